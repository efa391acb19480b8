// Batch-invariant attention over a unified paged KV store (decode and causal prefill).
//
// Sources: "Defeating Nondeterminism in LLM Inference" technical summary
// (mobiles-han blog), section 対応策：バッチ不変なカーネル設計, kernel table, row
// Attention — join the cache and the current tokens into one layout before
// attending, and cut the KV sequence into splits of a fixed SIZE (not a fixed
// count chosen from the batch); the usage article, section 注意点・補足実装
// (FixedAttention sketch: concatenate cache and new keys, fixed chunk size).
//
// Per-row schedule (identical for decode and prefill; a function of the row's own
// visible length L only):
//   * the visible keys 0..L-1 are cut into splits at absolute positions 0, 256,
//     512, ...; split s covers pages 16s .. 16s+15 of the row's page-table row;
//   * one warp reduces one (row, kv-head, split) for the Hq/Hkv query heads that
//     share the kv-head, page by page in ascending order, with an online softmax
//     in the base-2 domain (scores pre-multiplied by scale*log2(e));
//   * inside a page, a token's q.k is summed per lane over its DPL dims (DPL = 16
//     or 8, fixed by D and the group size) as two interleaved fp32 FMA chains (even
//     and odd dims, packed f32x2 FMAs) joined by one add, then by a fixed xor
//     reduce-scatter tree over the D/DPL lanes of the token; token t of the page
//     is handled by lane group t mod (32*DPL/D) and the groups' partial sums are
//     merged by a fixed xor tree at the end of the split;
//   * splits are folded in ascending order: M = max_s m_s, then
//     L = sum_s l_s 2^(m_s - M), O = sum_s o_s 2^(m_s - M) (FMA chains from 0),
//     out = O / L rounded to bf16.
// A prefill query at absolute position p is computed as a decode row of length
// p + 1 reading the same page-table row, so whole and chunked prefill, and decode,
// give the same bits for the same row. Slots past L are never folded in (stale
// slots may hold NaN); the copy engine only fetches the valid rows of a page.
#pragma once

#include "device.cuh"

namespace bi {
namespace attn {

constexpr int PAGE = BI_PAGE_TOKENS;
constexpr int SPLIT = BI_KV_SPLIT;
constexpr int PAGES_PER_SPLIT = SPLIT / PAGE;

// Where a query row reads its keys: decode rows use (row, seq_lens[row]);
// prefill rows use (q_seq[row], q_pos[row] + 1).
struct Rows {
  const int32_t* seq_lens;
  const int32_t* q_seq;
  const int32_t* q_pos;
  int num_pt_rows;
  int max_pages;
};

// Returns the row's visible length (0 if its ids are out of range, with the
// device error recorded) and its page-table row.
__device__ __forceinline__ int row_len(const Rows& R, int r, int& pt_row) {
  int len;
  if (R.q_pos) {
    pt_row = R.q_seq[r];
    len = R.q_pos[r] + 1;
  } else {
    pt_row = r;
    len = R.seq_lens[r];
  }
  if (pt_row < 0 || pt_row >= R.num_pt_rows || len < 0 || len > R.max_pages * PAGE) {
    record_error(BI_ERR_DEVICE_INDEX);
    pt_row = 0;
    return 0;
  }
  return len;
}

__device__ __forceinline__ int num_splits(const Rows& R, int r) {
  int pt_row;
  const int len = row_len(R, r, pt_row);
  return (len + SPLIT - 1) / SPLIT;
}

// off[r] = number of splits of rows 0..r-1; off[nrows] = total. One CTA of 1024 threads.
__global__ void __launch_bounds__(1024) split_offsets_kernel(Rows R, int nrows, int32_t* off) {
  __shared__ int32_t sums[1024];
  const int tid = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  const int per = (nrows + 1023) / 1024;
  const int r0 = tid * per;
  const int r1 = min(r0 + per, nrows);
  int local = 0;
  for (int r = r0; r < r1; ++r) local += num_splits(R, r);
  sums[tid] = local;
  __syncthreads();
  for (int d = 1; d < 1024; d <<= 1) {
    const int v = tid >= d ? sums[tid - d] : 0;
    __syncthreads();
    sums[tid] += v;
    __syncthreads();
  }
  int run = sums[tid] - local;
  for (int r = r0; r < r1; ++r) {
    off[r] = run;
    run += num_splits(R, r);
  }
  if (tid == 1023) off[nrows] = sums[1023];
}

// Reduce-scatter of G per-head partial sums over the LPT lanes of one token
// (xor butterfly, highest offset first). At each level a lane keeps the half of
// its heads selected by its lane bit and adds the partner's copy of that half
// (own + partner); once one head is left the remaining levels are all-reduce
// steps. Returns the full sum of head dl / (LPT / G).
template <int G, int LPT>
__device__ __forceinline__ float reduce_scatter(float (&v)[G], int dl) {
#pragma unroll
  for (int off = LPT / 2, n = G; off >= 1; off >>= 1) {
    if (n > 1) {
      const bool upper = (dl & off) != 0;
#pragma unroll
      for (int i = 0; i < G / 2; ++i) {
        if (i < n / 2) {
          const float send = upper ? v[i] : v[i + n / 2];
          const float keep = upper ? v[i + n / 2] : v[i];
          v[i] = __fadd_rn(keep, __shfl_xor_sync(kFullMask, send, off));
        }
      }
      n >>= 1;
    } else {
      v[0] = __fadd_rn(v[0], __shfl_xor_sync(kFullMask, v[0], off));
    }
  }
  return v[0];
}

// Inverse of the scatter: every lane of the token receives the G per-head values
// (head h held by lanes with dl / (LPT / G) == h). Pure data movement.
template <int G, int LPT>
__device__ __forceinline__ void all_gather(float x, int dl, float (&out)[G]) {
  out[0] = x;
#pragma unroll
  for (int off = LPT / G, n = 1; off < LPT; off <<= 1, n <<= 1) {
    const bool upper = (dl & off) != 0;
#pragma unroll
    for (int i = 0; i < G / 2; ++i) {
      if (i < n) {
        const float other = __shfl_xor_sync(kFullMask, out[i], off);
        const float mine = out[i];
        out[i] = upper ? other : mine;
        out[i + n] = upper ? mine : other;
      }
    }
  }
}

// Launch shape of the split kernel (a function of D and the group size G only):
// DPL dims per lane (16 when the registers allow it: fewer lanes per token, a
// shallower reduction tree), WARPS warps per CTA, each with its own ring of NST pages.
template <int D, int G>
struct SplitCfg {
  static constexpr int DPL = (D == 128 && G <= 4) ? 16 : 8;
  // 12 warps with 2-page rings where 16 dims per lane apply (measured on a B200 at
  // D = 128, group 4: 5-8 % more HBM bandwidth than 8 warps with 3-page rings at
  // B >= 4, same bits), 8 warps with 3-page rings otherwise
  static constexpr int WARPS = DPL == 16 ? 12 : 8;
  static constexpr int NST = DPL == 16 ? 2 : 3;
};

template <int D, int G>
constexpr int split_smem_bytes() {
  return SplitCfg<D, G>::WARPS * SplitCfg<D, G>::NST * (2 * PAGE * D * 2 + 8);
}

// The steps that reduce one (row, kv-head, split) for GW of the kv-head's G query
// heads on one warp: load the heads' query slices, fold pages, store the partials.
// The lane layout (SplitLanes) depends on D and G only, never on GW, and a head's
// q.k is summed by the same lanes in the same xor pairing whether its warp carries
// 1, 2, 4 or G heads (reduce_scatter pairs the same lanes at every level; a lane
// only drops the heads it does not keep), so a head's bits do not depend on GW.
//
// Lane layout: the LPT = D/DPL lanes of a token own DPL dims each, in 16-byte
// vectors v = 0..DPL/8-1 covering dims 8*(dl + v*LPT) .. +7 (interleaved so a
// quarter-warp's shared-memory reads are contiguous); TPW = 32/LPT tokens are
// processed per warp step, token t of a page by lane group t mod TPW.
template <int D, int G>
struct SplitLanes {
  static constexpr int DPL = SplitCfg<D, G>::DPL;
  static constexpr int NV = DPL / 8;   // 16-byte vectors per lane per token row
  static constexpr int LPT = D / DPL;  // lanes per token
  static constexpr int TPW = 32 / LPT; // tokens per warp step
  static constexpr int STEPS = PAGE / TPW;
  static constexpr int PAGE_BYTES = PAGE * D * 2;
  static constexpr int STAGE_BYTES = 2 * PAGE_BYTES;
};

// The lane's slice of query heads h0 .. h0+GW-1 of row r.
template <int D, int G, int GW>
__device__ __forceinline__ void load_q(const uint16_t* __restrict__ q, int64_t ldq, int r, int h0, int dl,
                                       float2 (&qf)[GW][SplitCfg<D, G>::DPL / 2]) {
  using T = SplitLanes<D, G>;
#pragma unroll
  for (int j = 0; j < GW; ++j)
#pragma unroll
    for (int v = 0; v < T::NV; ++v) {
      const uint4 qv = __ldg(reinterpret_cast<const uint4*>(q + (int64_t)r * ldq + (int64_t)(h0 + j) * D +
                                                            8 * (dl + v * T::LPT)));
      unpack8x2(qv, &qf[j][4 * v]);
    }
}

// Folds one page (K at kb, V at vb in shared memory, its first nvalid tokens
// visible) into the running (m, l, o) of the lane's head: scores, the base-2
// online-softmax rescale, then p * V. FULL: all PAGE tokens are visible (the same
// arithmetic without the visibility tests).
template <int D, int G, int GW, bool FULL = false>
__device__ __forceinline__ void fold_page(const float2 (&qf)[GW][SplitCfg<D, G>::DPL / 2], uint32_t kb, uint32_t vb,
                                          int nvalid, float c, int tg, int dl, float& m, float& l,
                                          float2 (&o)[GW][SplitCfg<D, G>::DPL / 2]) {
  using T = SplitLanes<D, G>;
  constexpr int NV = T::NV, LPT = T::LPT, TPW = T::TPW, STEPS = T::STEPS, DPL = T::DPL;
  // scores of this page: lane holds the score of its token for its head
  float sc[STEPS];
#pragma unroll
  for (int u = 0; u < STEPS; ++u) {
    const int t = u * TPW + tg;
    // two interleaved FMA chains per head (even / odd dims of the slice), then one add
    float2 acc[GW];
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      float2 kf[4];
      unpack8x2(ld_shared_v4(kb + (uint32_t)((t * D + 8 * (dl + v * LPT)) * 2)), kf);
#pragma unroll
      for (int i = 0; i < GW; ++i) {
        float2 a = v == 0 ? __fmul2_rn(qf[i][0], kf[0]) : __ffma2_rn(qf[i][4 * v], kf[0], acc[i]);
#pragma unroll
        for (int e = 1; e < 4; ++e) a = __ffma2_rn(qf[i][4 * v + e], kf[e], a);
        acc[i] = a;
      }
    }
    float part[GW];
#pragma unroll
    for (int i = 0; i < GW; ++i) part[i] = __fadd_rn(acc[i].x, acc[i].y);
    const float dot = reduce_scatter<GW, LPT>(part, dl);
    sc[u] = (FULL || t < nvalid) ? __fmul_rn(dot, c) : -INFINITY;
  }
  float pm = sc[0];
#pragma unroll
  for (int u = 1; u < STEPS; ++u) pm = fmaxf(pm, sc[u]);
#pragma unroll
  for (int o2 = LPT; o2 < 32; o2 <<= 1) pm = fmaxf(pm, __shfl_xor_sync(kFullMask, pm, o2));
  const float m_new = fmaxf(m, pm);
  const float alpha = m_new == -INFINITY ? 1.f : exp2f(__fsub_rn(m, m_new));
  // rescale the running sums; skipped when no head's max moved (x * 1 == x exactly)
  if (!__all_sync(kFullMask, alpha == 1.f)) {
    l = __fmul_rn(l, alpha);
    float al[GW];
    all_gather<GW, LPT>(alpha, dl, al);
#pragma unroll
    for (int i = 0; i < GW; ++i) {
      const float2 a2 = make_float2(al[i], al[i]);
#pragma unroll
      for (int e = 0; e < DPL / 2; ++e) o[i][e] = __fmul2_rn(o[i][e], a2);
    }
  }
#pragma unroll
  for (int u = 0; u < STEPS; ++u) {
    const int t = u * TPW + tg;
    const bool valid = FULL || t < nvalid;
    const float p = valid ? exp2f(__fsub_rn(sc[u], m_new)) : 0.f;
    l = __fadd_rn(l, p);
    float pa[GW];
    all_gather<GW, LPT>(p, dl, pa);
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      float2 vf[4];
      unpack8x2(ld_shared_v4(vb + (uint32_t)((t * D + 8 * (dl + v * LPT)) * 2)), vf);
      if (valid) {
#pragma unroll
        for (int i = 0; i < GW; ++i) {
          const float2 p2 = make_float2(pa[i], pa[i]);
#pragma unroll
          for (int e = 0; e < 4; ++e) o[i][4 * v + e] = __ffma2_rn(p2, vf[e], o[i][4 * v + e]);
        }
      }
    }
  }
  m = m_new;
}

// Merges the warp's token groups (fixed xor tree) and writes split slot f's
// unnormalised o[D] and (m, l) for query heads h0 .. h0+GW-1.
template <int D, int G, int GW>
__device__ __forceinline__ void store_split(float m, float l, float2 (&o)[GW][SplitCfg<D, G>::DPL / 2], int tg,
                                            int dl, int f, int Hq, int h0, float* __restrict__ po,
                                            float2* __restrict__ pml) {
  using T = SplitLanes<D, G>;
  constexpr int NV = T::NV, LPT = T::LPT, DPL = T::DPL, HEAD_LANES = LPT / GW;
#pragma unroll
  for (int o2 = LPT; o2 < 32; o2 <<= 1) {
    l = __fadd_rn(l, __shfl_xor_sync(kFullMask, l, o2));
#pragma unroll
    for (int i = 0; i < GW; ++i)
#pragma unroll
      for (int e = 0; e < DPL / 2; ++e) {
        const float2 other = make_float2(__shfl_xor_sync(kFullMask, o[i][e].x, o2),
                                         __shfl_xor_sync(kFullMask, o[i][e].y, o2));
        o[i][e] = __fadd2_rn(o[i][e], other);
      }
  }
  if (tg == 0) {
#pragma unroll
    for (int i = 0; i < GW; ++i)
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        float4* dst = reinterpret_cast<float4*>(po + ((int64_t)f * Hq + h0 + i) * D + 8 * (dl + v * LPT));
        dst[0] = make_float4(o[i][4 * v + 0].x, o[i][4 * v + 0].y, o[i][4 * v + 1].x, o[i][4 * v + 1].y);
        dst[1] = make_float4(o[i][4 * v + 2].x, o[i][4 * v + 2].y, o[i][4 * v + 3].x, o[i][4 * v + 3].y);
      }
    if (dl % HEAD_LANES == 0) pml[(int64_t)f * Hq + h0 + dl / HEAD_LANES] = make_float2(m, l);
  }
}

// Per-warp ring state of the split kernel: pages consumed so far (the ring position)
// and, for lane 0, the stages it filled and their phase parities (for drain_copies).
struct RingState {
  uint32_t seq, issued, ph_bits;
};

// The split kernel's work loop for GW query heads per warp over the (split slot,
// kv-head) items [begin, end): work units are (item, head part hp) with heads
// g*G + hp*GW .. +GW-1, dealt across CTAs first (unit = begin * HP + warp * gridDim.x
// + CTA + k * slots) so that fewer units than warp slots spread over every SM.
// Returns false if a copy never landed.
template <int D, int G, int GW>
__device__ __forceinline__ bool split_items(const uint16_t* __restrict__ q, int64_t ldq, int Hq, int Hkv,
                                            const uint16_t* __restrict__ kc, const uint16_t* __restrict__ vc,
                                            int64_t num_pages, const int32_t* __restrict__ pt, const Rows& R,
                                            int nrows, const int32_t* __restrict__ off, float* __restrict__ po,
                                            float2* __restrict__ pml, float c, int begin, int end, uint32_t ring,
                                            uint32_t bars, RingState& rs) {
  using T = SplitLanes<D, G>;
  constexpr int DPL = T::DPL, LPT = T::LPT, PAGE_BYTES = T::PAGE_BYTES, STAGE_BYTES = T::STAGE_BYTES;
  constexpr int WARPS = SplitCfg<D, G>::WARPS, NST = SplitCfg<D, G>::NST, HP = G / GW;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tg = lane / LPT, dl = lane % LPT;
  const int64_t kv_head_stride = (int64_t)PAGE * D;
  for (int item = begin * HP + warp * gridDim.x + blockIdx.x; item < end * HP; item += gridDim.x * WARPS) {
    const int fg = item / HP, hp = item - (item / HP) * HP;
    const int f = fg / Hkv, g = fg - (fg / Hkv) * Hkv;
    const int h0 = g * G + hp * GW;
    int lo = 0, hi = nrows;  // off[lo] <= f < off[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (off[mid] <= f) lo = mid;
      else hi = mid;
    }
    const int r = lo, s = f - off[lo];
    int pt_row;
    const int len = row_len(R, r, pt_row);
    const int t0 = s * SPLIT;
    const int t1 = min(t0 + SPLIT, len);
    const int np = (t1 - t0 + PAGE - 1) / PAGE;
    const int32_t* prow = pt + (int64_t)pt_row * R.max_pages + s * PAGES_PER_SPLIT;

    float2 qf[GW][DPL / 2];  // dims (2e, 2e+1) of the lane's slice in pair e
    load_q<D, G, GW>(q, ldq, r, h0, dl, qf);

    // Lane 0 starts the copy of page j of this split into its ring stage.
    auto issue = [&](int j, uint32_t sq) {
      const uint32_t st = sq % NST;
      const uint32_t bar = bars + 8 * st;
      const int pg = prow[j];
      const int nvalid = min(PAGE, t1 - t0 - j * PAGE);
      note_fill(rs.issued, rs.ph_bits, (int)st, (sq / NST) & 1u);
      if (pg < 0 || pg >= num_pages) {
        record_error(BI_ERR_DEVICE_INDEX);
        mbar_arrive_expect_tx(bar, 0);
        return;
      }
      const uint32_t bytes = (uint32_t)(nvalid * D * 2);
      const int64_t src = ((int64_t)pg * Hkv + g) * kv_head_stride;
      const uint32_t kdst = ring + st * STAGE_BYTES;
      mbar_arrive_expect_tx(bar, 2 * bytes);
      bulk_g2s(kdst, kc + src, bytes, bar);
      bulk_g2s(kdst + PAGE_BYTES, vc + src, bytes, bar);
    };
    if (lane == 0) {
      fence_proxy_async_smem();
      for (int j = 0; j < NST && j < np; ++j) issue(j, rs.seq + j);
    }

    float m = -INFINITY, l = 0.f;
    float2 o[GW][DPL / 2];
#pragma unroll
    for (int j = 0; j < GW; ++j)
#pragma unroll
      for (int e = 0; e < DPL / 2; ++e) o[j][e] = make_float2(0.f, 0.f);

    for (int j = 0; j < np; ++j, ++rs.seq) {
      const uint32_t st = rs.seq % NST;
      if (!__all_sync(kFullMask, mbar_wait(bars + 8 * st, (rs.seq / NST) & 1u))) return false;
      const int pg = prow[j];
      const int nvalid = (pg < 0 || pg >= num_pages) ? 0 : min(PAGE, t1 - t0 - j * PAGE);
      const uint32_t kb = ring + st * STAGE_BYTES;
      // warps carrying part of a kv-head's query heads (batches that leave warp slots
      // idle) have registers to spare for a second copy of the fold without the
      // visibility tests; the all-heads path keeps one copy (a second one spills)
      if (GW < G && nvalid == PAGE)
        fold_page<D, G, GW, true>(qf, kb, kb + PAGE_BYTES, PAGE, c, tg, dl, m, l, o);
      else
        fold_page<D, G, GW, false>(qf, kb, kb + PAGE_BYTES, nvalid, c, tg, dl, m, l, o);
      __syncwarp();
      if (lane == 0 && j + NST < np) {
        fence_proxy_async_smem();
        issue(j + NST, rs.seq + NST);
      }
    }
    store_split<D, G, GW>(m, l, o, tg, dl, f, Hq, h0, po, pml);
  }
  return true;
}

// One warp per (row, kv-head g, split) -- or per (row, kv-head, split, half or quarter
// of the G query heads) for the items of the last, partly filled round of warp slots
// when 2 or 4 times as many units still fit in one round: writes the split's (m, l)
// and unnormalised o[D] per query head into the workspace. Items that fill whole
// rounds keep their G heads on one warp (the fewest instructions per byte); a tail of
// fewer items than slots is cut finer so that it does not cost a full round. Each
// warp streams its split's pages through its own ring of NST stages. How the heads
// are spread over warps is a launch shape: every head's arithmetic is the same (see
// split_items).
template <int D, int G>
__global__ void __launch_bounds__(SplitCfg<D, G>::WARPS * 32, 1)
    attn_split_kernel(const uint16_t* __restrict__ q, int64_t ldq, int Hq, int Hkv, const uint16_t* __restrict__ kc,
                      const uint16_t* __restrict__ vc, int64_t num_pages, const int32_t* __restrict__ pt,
                      Rows R, int nrows, const int32_t* __restrict__ off, float* __restrict__ po,
                      float2* __restrict__ pml, float c) {
  using T = SplitLanes<D, G>;
  constexpr int LPT = T::LPT, STAGE_BYTES = T::STAGE_BYTES;
  constexpr int WARPS = SplitCfg<D, G>::WARPS, NST = SplitCfg<D, G>::NST;
  static_assert(G >= 1 && G <= LPT, "group size");

  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t ring = smem_u32(smem) + (uint32_t)(warp * NST * STAGE_BYTES);
  const uint32_t bars = smem_u32(smem) + (uint32_t)(WARPS * NST * STAGE_BYTES + warp * NST * 8);

  if (lane == 0) {
    for (int s = 0; s < NST; ++s) mbar_init(bars + 8 * s, 1);
    fence_mbar_init();
  }
  __syncwarp();
  pdl_wait();  // the offsets (and the caller's q and K/V) are complete from here on
  pdl_trigger();

  const int total = off[nrows] * Hkv;  // (split slot, kv-head) items
  const int64_t slots = (int64_t)gridDim.x * WARPS;
  const int full = (int)(total / slots * slots);  // items of the whole rounds
  const int tail = total - full;
  const int hs = (G >= 4 && tail > 0 && (int64_t)tail * 4 <= slots)   ? 4
                 : (G >= 2 && tail > 0 && (int64_t)tail * 2 <= slots) ? 2
                                                                      : 1;
  const int whole = hs == 1 ? total : full;  // items reduced with G heads per warp
  RingState rs{0u, 0u, 0u};
  bool ok = whole == 0 || split_items<D, G, G>(q, ldq, Hq, Hkv, kc, vc, num_pages, pt, R, nrows, off, po, pml, c, 0,
                                               whole, ring, bars, rs);
  if (ok && hs == 4)
    ok = split_items<D, G, (G >= 4 ? G / 4 : G)>(q, ldq, Hq, Hkv, kc, vc, num_pages, pt, R, nrows, off, po, pml, c,
                                                 full, total, ring, bars, rs);
  else if (ok && hs == 2)
    ok = split_items<D, G, (G >= 2 ? G / 2 : G)>(q, ldq, Hq, Hkv, kc, vc, num_pages, pt, R, nrows, off, po, pml, c,
                                                 full, total, ring, bars, rs);
  if (!ok) {  // a copy never landed: error recorded; let this warp's other copies land, then leave
    if (lane == 0) drain_copies(bars, 8, rs.issued, rs.ph_bits);
    __syncwarp();
  }
}

// Fold a row's splits in ascending order: one warp per (row, query head, group of
// 32 * DPL output dims), DPL dims per lane. The maximum of the splits' running maxima
// is taken lane-parallel, 128 splits per round trip (a maximum is exact in any order);
// lane j computes the weight of split j of each chunk of 32 and the weights are
// broadcast, so that every output dim and the normaliser are each one FMA chain in
// split order whatever DPL is. The splits are folded in groups of U = 32 / DPL; with
// one dim per lane (few rows) a group's partial outputs are loaded one group ahead
// (two register buffers) and each chunk's (m, l) one chunk ahead, so the fold waits
// for memory about once per row; with more dims per lane (many rows) one buffer keeps
// the registers low and the occupancy high. DPL only sets how many warps share a row:
// 1 when the batch gives few (row, head) pairs, D / 32 when it gives enough warps to
// fill the GPU.
template <int D, int DPL>
__global__ void __launch_bounds__(256, DPL == 1 ? 1 : 4) attn_combine_kernel(const float* __restrict__ po,
                                                           const float2* __restrict__ pml,
                                                           const int32_t* __restrict__ off, int nrows,
                                                           int Hq, uint16_t* __restrict__ out) {
  static_assert(DPL == 1 || DPL == 2 || DPL == 4, "dims per lane");
  static_assert(D % (32 * DPL) == 0, "a warp covers whole groups of dims");
  constexpr int NG = D / (32 * DPL);  // warps per (row, query head)
  constexpr int U = 32 / DPL;         // splits per group
  const int w = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  pdl_wait();  // the split partials are complete from here on
  pdl_trigger();
  if (w >= nrows * Hq * NG) return;
  const int rh = w / NG, g = w - (w / NG) * NG;
  const int r = rh / Hq, h = rh - (rh / Hq) * Hq;
  const int f0 = off[r], n = off[r + 1] - off[r];
  const int d0 = (g * 32 + lane) * DPL;
  const float2* ml_row = pml + (int64_t)f0 * Hq + h;             // split s at s * Hq
  const float* po_row = po + ((int64_t)f0 * Hq + h) * D + d0;    // split s at s * Hq * D
  const int64_t po_step = (int64_t)Hq * D;
  float M = -INFINITY;
  for (int s0 = 0; s0 < n; s0 += 128) {
    float mv[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int sp = s0 + c * 32 + lane;
      mv[c] = sp < n ? ml_row[(int64_t)sp * Hq].x : -INFINITY;
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) M = fmaxf(M, mv[c]);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float O[DPL];
#pragma unroll
  for (int d = 0; d < DPL; ++d) O[d] = 0.f;
  float L = 0.f;
  if (M != -INFINITY) {
    // the partial outputs of group gi (splits gi*U .. gi*U+U-1; past n: split 0 again, unused)
    auto load_group = [&](int gi, float (&v)[U][DPL]) {
#pragma unroll
      for (int j = 0; j < U; ++j) {
        const int sp = gi * U + j;
        const float* src = po_row + (int64_t)(sp < n ? sp : 0) * po_step;
        if constexpr (DPL == 4) {
          const float4 q = *reinterpret_cast<const float4*>(src);
          v[j][0] = q.x; v[j][1] = q.y; v[j][2] = q.z; v[j][3] = q.w;
        } else if constexpr (DPL == 2) {
          const float2 q = *reinterpret_cast<const float2*>(src);
          v[j][0] = q.x; v[j][1] = q.y;
        } else {
          v[j][0] = *src;
        }
      }
    };
    auto load_ml = [&](int chunk) {
      const int sp = chunk * 32 + lane;
      return sp < n ? ml_row[(int64_t)sp * Hq] : make_float2(-INFINITY, 0.f);
    };
    float2 ml = load_ml(0), ml_next = load_ml(1);
    float wl = lane < n ? exp2f(__fsub_rn(ml.x, M)) : 0.f;
    // fold group gi from buffer v (its chunk's weights are in wl / ml.y)
    auto fold_group = [&](int gi, const float (&v)[U][DPL]) {
#pragma unroll
      for (int j = 0; j < U; ++j) {
        const int sp = gi * U + j;
        const float wk = __shfl_sync(0xffffffffu, wl, sp & 31);
        const float lk = __shfl_sync(0xffffffffu, ml.y, sp & 31);
        if (sp < n) {
          L = __fmaf_rn(lk, wk, L);
#pragma unroll
          for (int d = 0; d < DPL; ++d) O[d] = __fmaf_rn(v[j][d], wk, O[d]);
        }
      }
      // the next group starts a new chunk of 32 splits: take its weights
      if (((gi + 1) * U) % 32 == 0) {
        const int chunk = (gi + 1) * U / 32;
        ml = ml_next;
        ml_next = load_ml(chunk + 1);
        const int sp = chunk * 32 + lane;
        wl = sp < n ? exp2f(__fsub_rn(ml.x, M)) : 0.f;
      }
    };
    const int ngroups = (n + U - 1) / U;
    if constexpr (DPL == 1) {
      // one dim per lane (few rows): the next group's loads overlap this group's fold
      float va[U][DPL], vb[U][DPL];
      load_group(0, va);
      for (int gi = 0; gi < ngroups; gi += 2) {
        if (gi + 1 < ngroups) load_group(gi + 1, vb);
        fold_group(gi, va);
        if (gi + 1 >= ngroups) break;
        if (gi + 2 < ngroups) load_group(gi + 2, va);
        fold_group(gi + 1, vb);
      }
    } else {
      // several dims per lane (many rows, e.g. prefill): one buffer, so that more warps
      // stay resident; other warps cover the loads
      float va[U][DPL];
      for (int gi = 0; gi < ngroups; ++gi) {
        load_group(gi, va);
        fold_group(gi, va);
      }
    }
  }
  float y[DPL];
#pragma unroll
  for (int d = 0; d < DPL; ++d) y[d] = L > 0.f ? __fdiv_rn(O[d], L) : 0.f;
  uint16_t* dst = out + (int64_t)rh * D + d0;
  if constexpr (DPL == 4) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]));
  } else if constexpr (DPL == 2) {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(y[0], y[1]);
  } else {
    *dst = to_bf16_bits(y[0]);
  }
}

// One warp per (token, kv-head): copy the token's K and V rows (row t of k_new /
// v_new starts at t * ld_new) into its page slot.
__global__ void __launch_bounds__(256) kv_append_kernel(const uint16_t* __restrict__ kn,
                                                        const uint16_t* __restrict__ vn, int64_t ld_new,
                                                        const int32_t* __restrict__ q_seq,
                                                        const int32_t* __restrict__ q_pos,
                                                        uint16_t* __restrict__ kc, uint16_t* __restrict__ vc,
                                                        int64_t num_pages, const int32_t* __restrict__ pt,
                                                        int num_seqs, int max_pages, int T, int Hkv, int D) {
  pdl_wait();  // inputs written by the previous kernel on the stream are complete from here on
  pdl_trigger();
  const int64_t w = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= (int64_t)T * Hkv) return;
  const int t = (int)(w / Hkv), g = (int)(w - (w / Hkv) * Hkv);
  const int sq = q_seq[t], pos = q_pos[t];
  if (sq < 0 || sq >= num_seqs || pos < 0 || pos >= max_pages * PAGE) {
    if (lane == 0) record_error(BI_ERR_DEVICE_INDEX);
    return;
  }
  const int pg = pt[(int64_t)sq * max_pages + pos / PAGE];
  if (pg < 0 || pg >= num_pages) {
    if (lane == 0) record_error(BI_ERR_DEVICE_INDEX);
    return;
  }
  const int64_t dst = (((int64_t)pg * Hkv + g) * PAGE + pos % PAGE) * D;
  const int64_t src = (int64_t)t * ld_new + (int64_t)g * D;
  for (int i = lane; i < D / 8; i += 32) {
    reinterpret_cast<uint4*>(kc + dst)[i] = __ldg(reinterpret_cast<const uint4*>(kn + src) + i);
    reinterpret_cast<uint4*>(vc + dst)[i] = __ldg(reinterpret_cast<const uint4*>(vn + src) + i);
  }
}

}  // namespace attn
}  // namespace bi
