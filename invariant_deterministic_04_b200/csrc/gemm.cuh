// Batch-invariant bf16 matmul C = A * W^T on 5th-generation tensor cores.
//
// Source: "Defeating Nondeterminism in LLM Inference" technical summary
// (mobiles-han blog), section 対応策：バッチ不変なカーネル設計, kernel table, row
// MatMul: use one kernel configuration for every shape — fixed tile sizes, no
// split-K, no switch between tensor-core and non-tensor-core paths — and accept a
// modest loss of speed.
//
// What fixes the bits of C[m, n]: the chain of tcgen05.mma.kind::f16 instructions
// (128 rows x BN columns x 16 k, A and B from shared memory, fp32 accumulator in
// tensor memory) that adds A[m, k0:k0+16] . W[n, k0:k0+16] for k0 = 0, 16, 32, ...
// in ascending order, then one round to bf16 (nearest even). Nothing else enters:
// no split-K, no second accumulator, no reduction across CTAs. The chain is the
// same for every M, for every position of row m inside its 128-row tile and for
// every position of column n inside its BN-wide tile; the GPU tests check both
// (a row alone equals the row at every tile position; every row of the M = 1..2048
// sweep equals the same row of the 2048-row product).
//
// The tile width BN (32, 64, 128, 192 or 256 columns) only decides how the N columns
// are dealt out to CTAs. A narrow tile gives many CTAs when M is small (each CTA then
// streams a thin slice of W, so more SMs pull W from HBM at once); a wide tile reads
// each A block from shared memory for more columns when M is large; 192 evens out the
// waves where 256 leaves SMs idle (N = 6144 at M = 512..1024: 8 % faster on a B200).
// The host picks the width from the tile counts (pick_bn); the width is not part of
// an element's arithmetic, so the choice cannot change a bit (tested over the sweep).
//
// Design (sm_100a):
//   * K is consumed in 64-wide blocks, each four 128xBNx16 MMAs in ascending k;
//   * A and W tiles come into shared memory by TMA (128-byte swizzle, K-major)
//     through an mbarrier ring (make_layout); a stage holds 1, 2 or 4 K blocks, so
//     that 4, 8 or 16 MMAs share one stage wait and one tcgen05.commit (the probe in
//     probes/mma_chain.cu measures that pair at about one MMA chain step); a ragged
//     tile's out-of-range rows and columns are zero-filled by TMA and masked in the
//     epilogue, so they cannot touch other rows;
//   * when M < 128 the A box holds only the first ceil8(M) rows; up to 64 rows the
//     A slot in shared memory holds only those rows too (more stages fit). Rows past
//     the box are never loaded: the MMAs read whatever lies there, and the result of
//     those rows lands in output rows >= M, which are never stored (row m of the
//     product depends on row m of A only);
//   * warp 0 issues TMA, warp 1 (one thread) issues the MMAs, warps 2-5 drain
//     TMEM (tcgen05.ld), round to bf16 (nearest even) and store; two TMEM
//     accumulators let the epilogue of one tile overlap the main loop of the next;
//   * persistent grid of min(#tiles, #SMs) CTAs; tile t goes to CTA t mod grid,
//     m-tiles of one W slice on neighbouring CTAs so the slice is read from HBM once;
//   * from 129 rows on, where the single-CTA tile would be 192 or 256 wide, clusters
//     of two CTAs compute 256 x 192 or 256 x 256 tiles with tcgen05.mma.cta_group::2
//     (gemm_bf16_pair_kernel; pick_pair): each CTA loads half of the tile's A rows and
//     half of its W rows, so a K block moves a third less into each SM's shared memory
//     (M = 2048, N = 14336, K = 4096 on a B200: 164 us against 182 us for 128 x 256
//     tiles, same bits);
//   * launched as a programmatic dependent of the previous kernel on the stream: the
//     barrier set-up, TMEM allocation and tensor-map prefetch overlap that kernel's
//     tail, and the TMA thread waits for it (pdl_wait) before the first load;
//   * every mbarrier wait is bounded; on expiry the kernel records
//     BI_ERR_DEVICE_TIMEOUT, all roles leave their loops, TMEM is freed.
#pragma once

#include <climits>
#include <mutex>

#include "device.cuh"

namespace bi {
namespace gemm {

constexpr int BM = 128, BK = 64;
constexpr int A_BYTES = BM * BK * 2;  // 16 KiB: a full 128-row A block
constexpr int kThreads = 192;         // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr int kEpiThreads = 128;
constexpr int kSmemBytes = 227 * 1024;   // dynamic shared memory of every launch
constexpr int kBarBytes = 8 * (2 * 32 + 4) + 16;  // barriers for up to 32 stages, TMEM slot, flag
constexpr int kMaxStages = 32;

// Tensor-memory columns allocated for two BN-wide fp32 accumulators: a power of two.
constexpr int tmem_cols_for(int bn) { return 2 * bn <= 32 ? 32 : 2 * bn <= 64 ? 64 : 2 * bn <= 128 ? 128 : 2 * bn <= 256 ? 256 : 512; }

template <int BN>
struct Cfg {
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "tcgen05 M=128 tile widths used here");
  static constexpr int B_BYTES = BN * BK * 2;   // BN rows of 128 bytes: whole 8-row swizzle atoms
  static constexpr int TMEM_COLS = tmem_cols_for(BN);  // two fp32 accumulators at columns 0 and BN
  // Instruction descriptor for kind::f16: D fp32 (bits 4-5 = 1), A bf16 (bits 7-9 =
  // 1), B bf16 (bits 10-12 = 1), both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
  static constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                    ((uint32_t)(BM >> 4) << 24);
};

// Stage ring of one launch (host-computed, a function of M and the tile width only):
// a K block is an A slot (the rows of the A box, 128 bytes each) followed by a W slot
// (BN rows); a stage holds kps consecutive K blocks; `stages` stages from the start of
// the (1024-aligned) dynamic shared memory, then `pad` bytes so that the MMA's 128-row
// read of the last A slot stays inside the allocation, then the barriers.
struct Layout {
  uint32_t a_slot, b_slot, kblk, kps, stages, stage_bytes, bar_offset;
};

// Shared-memory matrix descriptor for a K-major operand written by TMA with the
// 128-byte swizzle: rows of 128 bytes, 8-row atoms 1024 bytes apart (stride byte
// offset), version 1, layout SWIZZLE_128B (2). Start address is advanced by 32
// bytes per 16-element k step inside the atom.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Barrier layout shared by the kernels built on this main loop: full[0..S),
// empty[0..S), tfull[0..2), tempty[0..2), 8 bytes each from bar0.
struct Bars {
  uint32_t bar0;
  int stages;
  __device__ __forceinline__ uint32_t full(int s) const { return bar0 + 8u * (uint32_t)s; }
  __device__ __forceinline__ uint32_t empty(int s) const { return bar0 + 8u * (uint32_t)(stages + s); }
  __device__ __forceinline__ uint32_t tfull(int a) const { return bar0 + 8u * (uint32_t)(2 * stages + a); }
  __device__ __forceinline__ uint32_t tempty(int a) const { return bar0 + 8u * (uint32_t)(2 * stages + 2 + a); }
};

// Byte strides of the stage ring: compile-time with full 128-row A slots, from the
// host's Layout with compact A slots (the A box's rows).
template <int BN, int KPS, bool COMPACT>
struct Strides {
  uint32_t a_slot, kblk, stage;
  __device__ __forceinline__ explicit Strides(const Layout& L)
      : a_slot(COMPACT ? L.a_slot : (uint32_t)A_BYTES),
        kblk(COMPACT ? L.kblk : (uint32_t)(A_BYTES + Cfg<BN>::B_BYTES)),
        stage(COMPACT ? L.stage_bytes : (uint32_t)(KPS * (A_BYTES + Cfg<BN>::B_BYTES))) {}
};

// TMA producer (one thread): for every tile t = blockIdx.x, +gridDim.x, ... (m-tile
// t mod mt, n-tile t / mt) and every group of up to KPS 64-wide K blocks in ascending
// order, waits for a free stage and loads each K block's A rows and W rows into it.
// `issued` / `ph_bits` record the stages filled and their parities (drain_copies).
template <int BN, int KPS, bool COMPACT>
__device__ __forceinline__ void tma_producer(const CUtensorMap* tmA, const CUtensorMap* tmB, uint32_t base,
                                             const Layout& L, const Bars& bars, int tiles, int mt, int nkb,
                                             volatile int* abort_flag, uint32_t& issued, uint32_t& ph_bits) {
  const Strides<BN, KPS, COMPACT> S(L);
  const int stages = (int)L.stages;
  const uint32_t a_bytes = L.a_slot;  // bytes one A box brings (its rows x 128)
  int s = 0;
  uint32_t ph = 0;
  for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x) {
    const int m0 = (t % mt) * BM, n0 = (t / mt) * BN;
    for (int kb0 = 0; kb0 < nkb; kb0 += KPS) {
      const int nk = min(KPS, nkb - kb0);
      if (!mbar_wait(bars.empty(s), ph ^ 1u)) {
        *abort_flag = 1;
        break;
      }
      mbar_arrive_expect_tx(bars.full(s), (uint32_t)nk * (a_bytes + (uint32_t)Cfg<BN>::B_BYTES));
      const uint32_t st = base + (uint32_t)s * S.stage;
#pragma unroll
      for (int j = 0; j < KPS; ++j) {
        if (j < nk) {
          tma_load_2d(st + j * S.kblk, tmA, (kb0 + j) * BK, m0, bars.full(s));
          tma_load_2d(st + j * S.kblk + S.a_slot, tmB, (kb0 + j) * BK, n0, bars.full(s));
        }
      }
      note_fill(issued, ph_bits, s, ph);
      if (++s == stages) {
        s = 0;
        ph ^= 1u;
      }
    }
  }
}

// MMA issuer (one thread): per tile, waits for a free accumulator (two, BN columns
// apart in TMEM), then per stage for its data, and issues for each of its K blocks the
// four 128xBNx16 MMAs in ascending k; the first MMA of a tile overwrites the
// accumulator. A stage is released by one tcgen05.commit once all its MMAs have read
// it, an accumulator once its last MMA completes. The MMAs of an element are the same
// sequence whatever kps is: kps only sets how many of them share one wait and commit.
template <int BN, int KPS, bool COMPACT>
__device__ __forceinline__ void mma_issuer(uint32_t base, const Layout& L, const Bars& bars, uint32_t tmem, int tiles,
                                           int nkb, volatile int* abort_flag) {
  const Strides<BN, KPS, COMPACT> S(L);
  const int stages = (int)L.stages;
  int s = 0, acc = 0;
  uint32_t ph = 0, aph = 0;
  for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x) {
    if (!mbar_wait(bars.tempty(acc), aph ^ 1u)) {
      *abort_flag = 1;
      break;
    }
    tc_fence_after();
    const uint32_t d = tmem + (uint32_t)(acc * BN);
    bool ok = true;
    for (int kb0 = 0; kb0 < nkb; kb0 += KPS) {
      const int nk = min(KPS, nkb - kb0);
      if (!mbar_wait(bars.full(s), ph)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t st = base + (uint32_t)s * S.stage;
#pragma unroll
      for (int j = 0; j < KPS; ++j) {
        if (j < nk) {
          const uint32_t a = st + j * S.kblk, b = a + S.a_slot;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc_mma_f16(d, sw128_desc(a + kk * 32), sw128_desc(b + kk * 32), Cfg<BN>::IDESC,
                       ((kb0 + j) | kk) != 0 ? 1u : 0u);
        }
      }
      tc_commit(bars.empty(s));  // frees the stage once these MMAs have read it
      if (++s == stages) {
        s = 0;
        ph ^= 1u;
      }
    }
    if (!ok) {
      *abort_flag = 1;
      break;
    }
    tc_commit(bars.tfull(acc));  // accumulator complete
    acc ^= 1;
    if (acc == 0) aph ^= 1u;
  }
}

template <int BN, int KPS, bool COMPACT>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     uint16_t* __restrict__ C, int64_t ldc, int M, int N, int K, const Layout L) {
  using G = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const Bars bars{base + L.bar_offset, (int)L.stages};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L.bar_offset + 8 * (2 * L.stages + 4));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = (M + BM - 1) / BM, nt = (N + BN - 1) / BN;
  const int tiles = mt * nt;
  const int nkb = K / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < (int)L.stages; ++s) {
      mbar_init(bars.full(s), 1);
      mbar_init(bars.empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bars.tfull(a), 1);
      mbar_init(bars.tempty(a), kEpiThreads);
    }
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), G::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  uint32_t issued = 0, ph_bits = 0;  // the producer's filled stages and their phase parities

  if (threadIdx.x == 0) pdl_trigger();
  if (warp == 0) {
    // the previous kernel on the stream (which may write A or W, or read C) must be
    // done before the first load; the MMA and epilogue warps only follow the loads
    if (lane == 0) {
      pdl_wait();
      tma_producer<BN, KPS, COMPACT>(&tmA, &tmB, base, L, bars, tiles, mt, nkb, abort_flag, issued, ph_bits);
    }
  } else if (warp == 1) {
    if (lane == 0) mma_issuer<BN, KPS, COMPACT>(base, L, bars, tmem, tiles, nkb, abort_flag);
  } else {  // ---- epilogue: warps 2..5; warp w may read TMEM lanes 32*(w%4) .. +31
    const int quarter = warp & 3;
    int acc = 0;
    uint32_t aph = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
      const int m0 = (t % mt) * BM, n0 = (t / mt) * BN;
      const bool ok = __all_sync(kFullMask, mbar_wait(bars.tfull(acc), aph));
      if (!ok || *abort_flag) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const int row = m0 + quarter * 32 + lane;
      uint16_t* crow = C + (int64_t)row * ldc;
      const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        __syncwarp();  // tcgen05.ld is .sync.aligned: the warp must be converged
        tmem_ld_32x32b_x32(tbase + (uint32_t)(c * 32), r);
        tmem_wait_ld();
        const int col = n0 + c * 32;
        if (row < M && col < N) {
          if (col + 32 <= N) {
            uint4* dst = reinterpret_cast<uint4*>(crow + col);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 o;
              o.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
              o.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
              o.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
              o.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
              dst[v] = o;
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (col + e < N) crow[col + e] = to_bf16_bits(__uint_as_float(r[e]));
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bars.tempty(acc));
      acc ^= 1;
      if (acc == 0) aph ^= 1u;
    }
  }
  tc_fence_before();
  __syncthreads();
  // after an abort, loads may still be landing in stages nobody waited for
  if (warp == 0 && lane == 0 && *abort_flag) drain_copies(bars.bar0, 8, issued, ph_bits);
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, G::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// CTA-pair variant for large M: a cluster of two CTAs computes a 256 x PBN tile with
// tcgen05.mma.cta_group::2 (M = 256, N = PBN, 16 k): CTA r of the pair holds A rows
// 128r .. 128r+127 and W rows (output columns) r*PBN/2 .. (r+1)*PBN/2-1 of the tile,
// and its tensor memory receives output rows 128r .. 128r+127, all PBN columns. Each
// element is still one chain of MMAs over k in ascending order (the pair instruction
// sums the same 16-wide k slices of the same row and column), so the bits equal the
// single-CTA kernel's. Per SM and K block the pair moves 16 KB of A and PBN/2 rows of
// W into shared memory, where a 128 x 256 single-CTA tile moves 16 KB + 256 rows.
//   * both CTAs' warp 0 loads its own halves into its own ring and counts the bytes on
//     the leader's (rank 0) full barrier; the leader arms that barrier with both CTAs'
//     bytes;
//   * the leader's warp 1 issues the pair MMAs and commits each stage to both CTAs'
//     empty barriers and each finished accumulator to both CTAs' tfull barriers;
//   * both CTAs' warps 2-5 drain their own tensor memory and arrive on the leader's
//     tempty barrier (256 arrivals);
//   * the pair meets at cluster barriers after set-up and before tensor memory is freed,
//     so neither CTA leaves while the other may still read its shared memory.
template <int PBN>
struct PairCfg {
  static_assert(PBN % 32 == 0 && PBN >= 64 && PBN <= 256, "pair tile width");
  static constexpr int W_ROWS = PBN / 2;                    // W rows one CTA loads per tile
  static constexpr int STAGE = A_BYTES + W_ROWS * BK * 2;   // multiple of 1024: SW128 atoms stay aligned
  static constexpr int STAGES = (kSmemBytes - 1024 - kBarBytes) / STAGE > 8 ? 8
                                                                             : (kSmemBytes - 1024 - kBarBytes) / STAGE;
  static constexpr int SMEM = 1024 + STAGES * STAGE + kBarBytes;
  // kind::f16, bf16 x bf16 -> fp32, both K-major; N >> 3 at bit 17, M >> 4 at bit 24
  static constexpr uint32_t IDESC =
      (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(PBN >> 3) << 17) | ((256u >> 4) << 24);
  static_assert(STAGE % 1024 == 0, "stage alignment");
  static_assert(STAGES >= 4 && SMEM <= kSmemBytes, "pair ring");
};

// Up to three products C_g = A W_g^T with the same A (M x K) in one launch of the pair
// kernel: their tiles form one list (product 0's, then 1's, then 2's), so the pairs run
// whole rounds over all of them instead of a short last round per product. Fields are
// picked by g with selects, not indexed, so the parameter block stays in constant memory.
struct PairProblems {
  uint16_t* C0;
  uint16_t* C1;
  uint16_t* C2;
  int64_t ldc0, ldc1, ldc2;
  int N0, N1, N2;
  int start1, start2, total;  // first tile of products 1 and 2; tiles in all
  int count;
};
constexpr int kMaxProblems = 3;

template <int PBN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_bf16_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                          const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmB2,
                          const PairProblems pp, int M, int K) {
  using P = PairCfg<PBN>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const Bars bars{base + (uint32_t)(P::STAGES * P::STAGE), P::STAGES};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + P::STAGES * P::STAGE + 8 * (2 * P::STAGES + 4));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = (int)blockIdx.x >> 1, npairs = (int)gridDim.x >> 1;
  const int mt = (M + 255) / 256;
  const int tiles = pp.total;
  // tile t: product g (the last whose first tile is <= t); within it, local tile u is
  // m-tile u % mt of W slice u / mt (the m-tiles of one slice on neighbouring pairs)
  auto product_of = [&](int t, int& u) -> int {
    const int g = (pp.count > 2 && t >= pp.start2) ? 2 : ((pp.count > 1 && t >= pp.start1) ? 1 : 0);
    u = t - (g == 2 ? pp.start2 : (g == 1 ? pp.start1 : 0));
    return g;
  };
  const int nkb = K / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < P::STAGES; ++s) {
      mbar_init(bars.full(s), 1);
      mbar_init(bars.empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bars.tfull(a), 1);
      mbar_init(bars.tempty(a), 2 * kEpiThreads);
    }
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB0);
    if (pp.count > 1) prefetch_tensormap(&tmB1);
    if (pp.count > 2) prefetch_tensormap(&tmB2);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_barrier();  // both CTAs' barriers are initialised and the pair's TMEM is allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) pdl_trigger();
  uint32_t issued = 0, ph_bits = 0;  // the leader's armed stages and their parities

  if (warp == 0) {
    if (lane == 0) {
      pdl_wait();  // the previous kernel on the stream is done before the first load
      int s = 0;
      uint32_t ph = 0;
      for (int t = pair; t < tiles && !*abort_flag; t += npairs) {
        int u;
        const int g = product_of(t, u);
        const CUtensorMap* tmB = g == 0 ? &tmB0 : (g == 1 ? &tmB1 : &tmB2);
        const int m0 = (u % mt) * 256 + (int)rank * 128, n0 = (u / mt) * PBN + (int)rank * P::W_ROWS;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(bars.empty(s), ph ^ 1u)) {
            *abort_flag = 1;
            break;
          }
          const uint32_t full_leader = map_to_rank(bars.full(s), 0);
          if (leader) {
            mbar_arrive_expect_tx(bars.full(s), 2u * (uint32_t)P::STAGE);
            note_fill(issued, ph_bits, s, ph);
          }
          const uint32_t st = base + (uint32_t)s * P::STAGE;
          tma_load_2d_pair(st, &tmA, kb * BK, m0, full_leader);
          tma_load_2d_pair(st + A_BYTES, tmB, kb * BK, n0, full_leader);
          if (++s == P::STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      int s = 0, acc = 0;
      uint32_t ph = 0, aph = 0;
      for (int t = pair; t < tiles && !*abort_flag; t += npairs) {
        if (!mbar_wait(bars.tempty(acc), aph ^ 1u)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(acc * 256);
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(bars.full(s), ph)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = base + (uint32_t)s * P::STAGE, b = a + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc_mma_f16_pair(d, sw128_desc(a + kk * 32), sw128_desc(b + kk * 32), P::IDESC, (kb | kk) != 0 ? 1u : 0u);
          tc_commit_pair_mc(bars.empty(s), (uint16_t)0x3);  // both CTAs' stage s is free once read
          if (++s == P::STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) {
          *abort_flag = 1;
          break;
        }
        tc_commit_pair_mc(bars.tfull(acc), (uint16_t)0x3);  // both halves of the accumulator are complete
        acc ^= 1;
        if (acc == 0) aph ^= 1u;
      }
    }
  } else {  // ---- epilogue: warps 2..5 of both CTAs; warp w reads TMEM lanes 32*(w%4) .. +31
    const int quarter = warp & 3;
    const uint32_t tempty_leader0 = map_to_rank(bars.tempty(0), 0), tempty_leader1 = map_to_rank(bars.tempty(1), 0);
    int acc = 0;
    uint32_t aph = 0;
    for (int t = pair; t < tiles; t += npairs) {
      int u;
      const int g = product_of(t, u);
      uint16_t* const C = g == 0 ? pp.C0 : (g == 1 ? pp.C1 : pp.C2);
      const int64_t ldc = g == 0 ? pp.ldc0 : (g == 1 ? pp.ldc1 : pp.ldc2);
      const int N = g == 0 ? pp.N0 : (g == 1 ? pp.N1 : pp.N2);
      const int m0 = (u % mt) * 256 + (int)rank * 128, n0 = (u / mt) * PBN;
      const bool ok = __all_sync(kFullMask, mbar_wait(bars.tfull(acc), aph));
      if (!ok || *abort_flag) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const int row = m0 + quarter * 32 + lane;
      uint16_t* crow = C + (int64_t)row * ldc;
      const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * 256);
#pragma unroll 1
      for (int c = 0; c < PBN / 32; ++c) {
        uint32_t r[32];
        __syncwarp();  // tcgen05.ld is .sync.aligned: the warp must be converged
        tmem_ld_32x32b_x32(tbase + (uint32_t)(c * 32), r);
        tmem_wait_ld();
        const int col = n0 + c * 32;
        if (row < M && col < N) {
          if (col + 32 <= N) {
            uint4* dst = reinterpret_cast<uint4*>(crow + col);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 o;
              o.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
              o.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
              o.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
              o.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
              dst[v] = o;
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (col + e < N) crow[col + e] = to_bf16_bits(__uint_as_float(r[e]));
          }
        }
      }
      tc_fence_before();
      if (leader)
        mbar_arrive(bars.tempty(acc));
      else
        mbar_arrive_cluster(acc == 0 ? tempty_leader0 : tempty_leader1);
      acc ^= 1;
      if (acc == 0) aph ^= 1u;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && warp == 0 && lane == 0) {
    if (leader) {
      drain_copies(bars.bar0, 8, issued, ph_bits);  // the armed stages count both CTAs' copies
    } else {
      // this CTA's copies are counted on the leader's barriers: give any still in flight
      // a bounded time to land before the pair is released
      const uint64_t t0 = global_timer_ns();
      while (global_timer_ns() - t0 < 200000ull) {
      }
    }
  }
  __syncthreads();
  cluster_barrier();  // neither CTA leaves while the other's MMAs or copies may use its shared memory
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 tensor [rows, cols] with row stride ld (elements); box = 64 cols x box_rows.
inline bool make_map(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols, int64_t ld,
                     uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2u};
  cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Number of SMs of a device (cached; 0 if the query fails).
inline int device_sms(int dev) {
  static int sms[64];
  static std::mutex mu;
  if (dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (sms[dev] == 0 && cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    sms[dev] = 0;
  return sms[dev];
}

// Raises the dynamic shared-memory limit of kernel `fn` once per device and keeps
// the result, so that a failure is reported on every later call too.
template <typename F>
inline cudaError_t set_smem_once(F fn, int bytes, std::once_flag* once, cudaError_t* result, int dev) {
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::call_once(once[dev], [&] { result[dev] = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes); });
  return result[dev];
}

template <int BN, int KPS, bool COMPACT>
inline cudaError_t prepare(int dev) {
  static std::once_flag once[64];
  static cudaError_t result[64];
  return set_smem_once(gemm_bf16_kernel<BN, KPS, COMPACT>, kSmemBytes, once, result, dev);
}

// Rows of A one stage loads: a whole 128-row block, or only ceil8(M) rows when the
// product has fewer than 128 rows.
inline uint32_t a_box_rows(int64_t M) { return M >= BM ? (uint32_t)BM : (uint32_t)((M + 7) / 8 * 8); }

// Tile width for an M x N product on `sms` SMs. Cost of one tile per 64-wide K
// block, in shared-memory cycles (128 bytes per cycle): the A box written by TMA,
// A read by the four MMAs, the W block written and read, i.e. rows + 128 + 2 BN.
// Tiles run in waves of `sms`; the width with the fewest cycles in total wins, ties
// to the wider tile (fewer re-reads of A from L2). A scheduling choice only.
inline int pick_bn(int64_t M, int64_t N, int sms) {
  if (sms <= 0) sms = 1;
  const int64_t mt = (M + BM - 1) / BM;
  const int64_t rows = a_box_rows(M);
  int best = 256;
  int64_t best_cost = INT64_MAX;
  for (int bn : {256, 192, 128, 64, 32}) {
    const int64_t tiles = mt * ((N + bn - 1) / bn);
    const int64_t waves = (tiles + sms - 1) / sms;
    const int64_t cost = waves * (rows + 128 + 2 * bn);
    if (cost < best_cost) {
      best_cost = cost;
      best = bn;
    }
  }
  return best;
}

// Width of the CTA-pair tile (256 rows x 256 or 192 columns) for an M x N product, or
// 0 for the single-CTA kernel. Pairs from 129 rows on (two 128-row m-tiles become one
// pair tile on as many SMs), where the single-CTA choice is a wide tile (192 or 256): a
// pair moves a third less into each SM's shared memory per K block. Of the two pair widths, the one with the lower cost of whole rounds of tiles
// over the pairs (sms / 2 clusters), a 256 x 192 tile costing 8/9 of a 256 x 256 one
// (as measured on a B200: the time of a tile falls more slowly than its width).
inline int pick_pair(int64_t M, int64_t N, int sms) {
  if (M <= 128 || pick_bn(M, N, sms) < 192) return 0;
  const int64_t pairs = sms / 2 > 0 ? sms / 2 : 1;
  const int64_t mt = (M + 255) / 256;
  const int64_t r256 = (mt * ((N + 255) / 256) + pairs - 1) / pairs;
  const int64_t r192 = (mt * ((N + 191) / 192) + pairs - 1) / pairs;
  return 8 * r192 < 9 * r256 ? 192 : 256;
}

// The stage ring for an M-row product with tile width bn. From 65 rows of A on: full
// 128-row A slots in 198 KB, two K blocks per stage where that leaves three stages
// (tile widths up to 128), else one (width 256: four stages). Up to 64 rows: the A
// slot holds only the rows of the A box, and the most K blocks per stage (4, else 2)
// that still leave three stages. Grouping K blocks lets 8 or 16 MMAs share one wait
// and one commit instead of 4; compact A slots leave room for more W in flight.
constexpr uint32_t kRingBudget = 198 * 1024;
inline Layout make_layout(int64_t M, int bn) {
  Layout L{};
  const uint32_t arows = a_box_rows(M);
  L.b_slot = (uint32_t)bn * BK * 2;
  if (arows > 64) {
    L.a_slot = arows * BK * 2;  // the A box's bytes; its slot is a full 16 KiB
    L.kblk = (uint32_t)A_BYTES + L.b_slot;
    L.kps = kRingBudget / (2 * L.kblk) >= 3 ? 2 : 1;
    L.stage_bytes = L.kps * L.kblk;
    L.stages = kRingBudget / L.stage_bytes;
    L.bar_offset = L.stages * L.stage_bytes;
    return L;
  }
  L.a_slot = arows * BK * 2;
  L.kblk = L.a_slot + L.b_slot;
  const uint32_t pad = (uint32_t)A_BYTES - L.a_slot;  // the MMA reads 128 rows from every A slot
  const uint32_t ring = (uint32_t)kSmemBytes - 1024 - kBarBytes - pad;
  for (uint32_t kps : {4u, 2u, 1u}) {
    L.kps = kps;
    L.stage_bytes = kps * L.kblk;
    L.stages = ring / L.stage_bytes;
    if (L.stages >= 3) break;
  }
  if (L.stages > (uint32_t)kMaxStages) L.stages = kMaxStages;
  L.bar_offset = (L.stages * L.stage_bytes + pad + 7u) & ~7u;
  return L;
}

template <int BN, int KPS, bool COMPACT>
inline bi_status launch_kps(const uint16_t* A, int64_t lda, const uint16_t* W, int64_t ldw, uint16_t* C, int64_t ldc,
                            int64_t M, int64_t N, int64_t K, const Layout& L, int dev, int sms, cudaStream_t st) {
  if (prepare<BN, KPS, COMPACT>(dev) != cudaSuccess) return BI_ERR_CUDA;
  CUtensorMap ta, tb;
  if (!make_map(&ta, A, M, K, lda, a_box_rows(M)) || !make_map(&tb, W, N, K, ldw, BN)) return BI_ERR_CUDA;
  const int64_t tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int grid = (int)(tiles < sms ? tiles : sms);
  const int smem = (int)(1024 + L.bar_offset + kBarBytes);
  return launch_pdl(gemm_bf16_kernel<BN, KPS, COMPACT>, dim3(grid), dim3(kThreads), (size_t)smem, st, ta, tb, C, ldc,
                    (int)M, (int)N, (int)K, L) == cudaSuccess
             ? BI_OK
             : BI_ERR_CUDA;
}

// The CTA-pair kernel with tile width PBN: one cluster of two CTAs per 256 x PBN tile
// at a time, as many clusters as can be resident at once (queried once per device: a
// cluster's two CTAs share a GPC, so odd SM counts per GPC can leave an SM out).
template <int PBN>
inline int pair_clusters(int dev) {
  using P = PairCfg<PBN>;
  static std::once_flag once[64];
  static int clusters[64];
  if (dev < 0 || dev >= 64) return 0;
  std::call_once(once[dev], [&] {
    int n = 0;
    if (cudaFuncSetAttribute(gemm_bf16_pair_kernel<PBN>, cudaFuncAttributeMaxDynamicSharedMemorySize, P::SMEM) ==
        cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2);
      cfg.blockDim = dim3(kThreads);
      cfg.dynamicSmemBytes = P::SMEM;
      if (cudaOccupancyMaxActiveClusters(&n, gemm_bf16_pair_kernel<PBN>, &cfg) != cudaSuccess) n = 0;
    }
    clusters[dev] = n > 0 ? n : 0;
  });
  return clusters[dev];
}

template <int BN>
inline bi_status launch_bn(const uint16_t* A, int64_t lda, const uint16_t* W, int64_t ldw, uint16_t* C,
                           int64_t ldc, int64_t M, int64_t N, int64_t K, int dev, int sms, cudaStream_t st) {
  const Layout L = make_layout(M, BN);
  if (L.stages < 2) return BI_ERR_UNSUPPORTED;
  if (a_box_rows(M) > 64)
    return L.kps == 2 ? launch_kps<BN, 2, false>(A, lda, W, ldw, C, ldc, M, N, K, L, dev, sms, st)
                      : launch_kps<BN, 1, false>(A, lda, W, ldw, C, ldc, M, N, K, L, dev, sms, st);
  if (L.kps == 4) return launch_kps<BN, 4, true>(A, lda, W, ldw, C, ldc, M, N, K, L, dev, sms, st);
  if (L.kps == 2) return launch_kps<BN, 2, true>(A, lda, W, ldw, C, ldc, M, N, K, L, dev, sms, st);
  return launch_kps<BN, 1, true>(A, lda, W, ldw, C, ldc, M, N, K, L, dev, sms, st);
}

// An M x N product on CTA pairs with tile width PBN: one cluster of two CTAs per
// 256 x PBN tile at a time, as many clusters as can be resident at once. Tiles of the
// last round (fewer than the pairs) are not cut up: a dependent pair MMA takes about as
// long at any width (narrower tiles for that round, or handing its tiles to the
// single-CTA kernel in a second launch, measured no faster on a B200).
// One product of a multi-product launch: C = A W^T, W [N, K] with row stride ldw.
struct Product {
  const uint16_t* W;
  int64_t ldw;
  uint16_t* C;
  int64_t ldc;
  int64_t N;
};

template <int PBN>
inline bi_status launch_pair(const uint16_t* A, int64_t lda, const Product* prods, int count, int64_t M, int64_t K,
                             int dev, cudaStream_t st) {
  const int clusters = pair_clusters<PBN>(dev);
  if (clusters <= 0) return BI_ERR_CUDA;
  if (count < 1 || count > kMaxProblems) return BI_ERR_SHAPE;
  CUtensorMap ta, tb[kMaxProblems];
  if (!make_map(&ta, A, M, K, lda, 128)) return BI_ERR_CUDA;
  const int64_t mt = (M + 255) / 256;
  int64_t start[kMaxProblems + 1] = {0, 0, 0, 0};
  for (int g = 0; g < count; ++g) {
    if (!make_map(&tb[g], prods[g].W, prods[g].N, K, prods[g].ldw, PBN / 2)) return BI_ERR_CUDA;
    start[g + 1] = start[g] + mt * ((prods[g].N + PBN - 1) / PBN);
  }
  for (int g = count; g < kMaxProblems; ++g) {
    tb[g] = tb[0];
    start[g + 1] = start[g];
  }
  if (start[count] > INT_MAX / 2) return BI_ERR_SHAPE;
  const Product& p1 = prods[count > 1 ? 1 : 0];
  const Product& p2 = prods[count > 2 ? 2 : 0];
  PairProblems pp{};
  pp.C0 = prods[0].C;
  pp.C1 = p1.C;
  pp.C2 = p2.C;
  pp.ldc0 = prods[0].ldc;
  pp.ldc1 = p1.ldc;
  pp.ldc2 = p2.ldc;
  pp.N0 = (int)prods[0].N;
  pp.N1 = (int)p1.N;
  pp.N2 = (int)p2.N;
  pp.start1 = (int)start[1];
  pp.start2 = (int)start[2];
  pp.total = (int)start[count];
  pp.count = count;
  const int pairs = (int)(pp.total < clusters ? pp.total : clusters);
  return launch_pdl(gemm_bf16_pair_kernel<PBN>, dim3(2 * pairs), dim3(kThreads), (size_t)PairCfg<PBN>::SMEM, st,
                    ta, tb[0], tb[1], tb[2], pp, (int)M, (int)K) == cudaSuccess
             ? BI_OK
             : BI_ERR_CUDA;
}

// bn: tile width (0 = pick_bn's choice for this device).
inline bi_status launch(const uint16_t* A, int64_t lda, const uint16_t* W, int64_t ldw, uint16_t* C,
                        int64_t ldc, int64_t M, int64_t N, int64_t K, cudaStream_t st, int bn = 0) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BI_ERR_CUDA;
  const int sms = device_sms(dev);
  if (sms <= 0) return BI_ERR_CUDA;
  if (bn == 0) {
    // large products: CTA pairs on 256-row tiles (the same element chains)
    switch (pick_pair(M, N, sms)) {
      case 256: {
        const Product p{W, ldw, C, ldc, N};
        return launch_pair<256>(A, lda, &p, 1, M, K, dev, st);
      }
      case 192: {
        const Product p{W, ldw, C, ldc, N};
        return launch_pair<192>(A, lda, &p, 1, M, K, dev, st);
      }
      default: bn = pick_bn(M, N, sms);
    }
  }
  switch (bn) {
    case 32: return launch_bn<32>(A, lda, W, ldw, C, ldc, M, N, K, dev, sms, st);
    case 64: return launch_bn<64>(A, lda, W, ldw, C, ldc, M, N, K, dev, sms, st);
    case 128: return launch_bn<128>(A, lda, W, ldw, C, ldc, M, N, K, dev, sms, st);
    case 192: return launch_bn<192>(A, lda, W, ldw, C, ldc, M, N, K, dev, sms, st);
    case 256: return launch_bn<256>(A, lda, W, ldw, C, ldc, M, N, K, dev, sms, st);
    default: return BI_ERR_UNSUPPORTED;
  }
}

// Several products with the same A: C_g = A W_g^T, g < count (at most kMaxProblems).
// When every product would run on CTA pairs alone (pick_pair), one launch of the pair
// kernel takes all their tiles in one list, with the tile width chosen the way
// pick_pair chooses it, from the joint tile counts; otherwise each product is its own
// launch. Either way each element is the same MMA chain as in a bi_matmul call alone.
inline bi_status launch_multi(const uint16_t* A, int64_t lda, const Product* prods, int count, int64_t M, int64_t K,
                              cudaStream_t st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BI_ERR_CUDA;
  const int sms = device_sms(dev);
  if (sms <= 0) return BI_ERR_CUDA;
  bool joint = count > 1;
  for (int g = 0; g < count && joint; ++g) joint = pick_pair(M, prods[g].N, sms) != 0;
  if (joint) {
    const int64_t pairs = sms / 2 > 0 ? sms / 2 : 1, mt = (M + 255) / 256;
    int64_t t256 = 0, t192 = 0;
    for (int g = 0; g < count; ++g) {
      t256 += mt * ((prods[g].N + 255) / 256);
      t192 += mt * ((prods[g].N + 191) / 192);
    }
    const int64_t r256 = (t256 + pairs - 1) / pairs, r192 = (t192 + pairs - 1) / pairs;
    return 8 * r192 < 9 * r256 ? launch_pair<192>(A, lda, prods, count, M, K, dev, st)
                               : launch_pair<256>(A, lda, prods, count, M, K, dev, st);
  }
  for (int g = 0; g < count; ++g) {
    const bi_status r = launch(A, lda, prods[g].W, prods[g].ldw, prods[g].C, prods[g].ldc, M, prods[g].N, K, st);
    if (r != BI_OK) return r;
  }
  return BI_OK;
}

}  // namespace gemm
}  // namespace bi
