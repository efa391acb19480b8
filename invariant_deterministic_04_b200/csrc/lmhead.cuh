// Greedy LM head with a selective FP32 recompute.
//
// Source: "Greedy Decoding Is Not Precision-Invariant: Cross-Precision Output
// Divergence in LLM Inference" (arXiv 2609.26621), abstract: whether greedy
// decoding flips depends mainly on the top-2 logit margin at the LM head; the best
// low-overhead fix recomputes the LM head in FP32 only when that margin is below a
// threshold.
//
// Pipeline (all on the caller's stream, no host round trip):
//   1. bf16 logits = bi_matmul(h, W)                         (tensor cores)
//   2. top2_kernel: per row, top-2 of the bf16 logits (value desc, index asc; NaN
//      never wins), margin = top1 - top2 in fp32, flag = margin < threshold;
//      token = top-1 index.
//   3. compact_kernel: ascending list of flagged rows.
//   4. recompute_kernel, or recompute_stream_kernel for few flagged rows: fp32
//      logits of the flagged rows from bf16 operands widened to fp32, each logit one
//      FMA chain over k = 0..K-1 (CUDA cores).
//   5. argmax_kernel: token of each flagged row = argmax of its fp32 logits.
// The top-2 and argmax merges are order-independent (a strict total order), and
// each fp32 logit depends only on its own row, so every row is batch-invariant.
#pragma once

#include <cstddef>

#include "device.cuh"

namespace bi {
namespace lmhead {

struct Top2 {
  float v1;
  int i1;
  float v2;
  int i2;
};

struct ArgBest {
  float v;
  int i;
};

__device__ __forceinline__ bool better(float a, int ia, float b, int ib) {
  return a > b || (a == b && ia < ib);
}

__device__ __forceinline__ void insert(Top2& t, float v, int i) {
  if (better(v, i, t.v1, t.i1)) {
    t.v2 = t.v1;
    t.i2 = t.i1;
    t.v1 = v;
    t.i1 = i;
  } else if (better(v, i, t.v2, t.i2)) {
    t.v2 = v;
    t.i2 = i;
  }
}

__device__ __forceinline__ float sanitize(float v) { return v != v ? -INFINITY : v; }

constexpr int kThreads = 256;
constexpr int kParts = 8;  // CTAs (one cluster) per row for the top-2 and the argmax

// Merge of a CTA's per-thread top-2 into thread 0 (warp butterfly, then warps in order).
__device__ __forceinline__ Top2 block_top2(Top2 t, Top2* warp_best) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const float a1 = __shfl_xor_sync(kFullMask, t.v1, o), a2 = __shfl_xor_sync(kFullMask, t.v2, o);
    const int j1 = __shfl_xor_sync(kFullMask, t.i1, o), j2 = __shfl_xor_sync(kFullMask, t.i2, o);
    insert(t, a1, j1);
    insert(t, a2, j2);
  }
  if ((threadIdx.x & 31) == 0) warp_best[threadIdx.x >> 5] = t;
  __syncthreads();
  Top2 b = warp_best[0];
  if (threadIdx.x == 0)
    for (int w = 1; w < kThreads / 32; ++w) {
      insert(b, warp_best[w].v1, warp_best[w].i1);
      insert(b, warp_best[w].v2, warp_best[w].i2);
    }
  return b;
}

// Per row, a cluster of kParts CTAs: part p scans vectors p * ceil(n/8) .. of the row's n
// 8-element vectors (a split fixed by V); CTA 0 merges the parts' top-2 through
// distributed shared memory. The top-2 under a strict total order is exact, so the split
// does not change it.
__global__ void __cluster_dims__(kParts, 1, 1) __launch_bounds__(kThreads)
    top2_kernel(const uint16_t* __restrict__ logits, int64_t V, float threshold, int32_t* __restrict__ tokens,
                int32_t* __restrict__ flags, unsigned int* __restrict__ ticket) {
  pdl_wait();  // inputs written by the previous kernel on the stream are complete from here on
  pdl_trigger();
  __shared__ Top2 warp_best[kThreads / 32];
  __shared__ Top2 part_best;
  const int64_t row = blockIdx.x / kParts;
  const uint32_t part = cluster_rank();
  if (blockIdx.x == 0 && threadIdx.x == 0 && ticket) *ticket = 0;  // for recompute_stream_kernel
  const uint4* src = reinterpret_cast<const uint4*>(logits + row * V);
  const int64_t nvec = V / 8, per = (nvec + kParts - 1) / kParts;
  const int64_t j0 = (int64_t)part * per, j1 = min(nvec, j0 + per);
  Top2 t{-INFINITY, 0x7FFFFFFF, -INFINITY, 0x7FFFFFFF};
  for (int64_t j = j0 + threadIdx.x; j < j1; j += kThreads) {
    float f[8];
    unpack8(__ldg(src + j), f);
#pragma unroll
    for (int e = 0; e < 8; ++e) insert(t, sanitize(f[e]), (int)(j * 8 + e));
  }
  const Top2 b = block_top2(t, warp_best);
  if (threadIdx.x == 0) part_best = b;
  cluster_barrier();  // every part's top-2 is in its shared memory
  if (part == 0 && threadIdx.x == 0) {
    Top2 m = part_best;
    for (uint32_t p = 1; p < kParts; ++p) {
      const uint32_t base = map_to_rank(smem_u32(&part_best), p);
      insert(m, ld_cluster_f32(base + offsetof(Top2, v1)), ld_cluster_s32(base + offsetof(Top2, i1)));
      insert(m, ld_cluster_f32(base + offsetof(Top2, v2)), ld_cluster_s32(base + offsetof(Top2, i2)));
    }
    const float margin = __fsub_rn(m.v1, m.v2);  // +inf when V == 1
    tokens[row] = m.i1;
    flags[row] = (margin < threshold) ? 1 : 0;
  }
  cluster_barrier();  // no part leaves while CTA 0 may still read its shared memory
}

// list[0..count) = indices of flagged rows, ascending; list[M] = count.
__global__ void __launch_bounds__(1024) compact_kernel(const int32_t* __restrict__ flags, int M,
                                                       int32_t* __restrict__ list) {
  pdl_wait();  // inputs written by the previous kernel on the stream are complete from here on
  pdl_trigger();
  __shared__ int32_t sums[1024];
  const int tid = threadIdx.x;
  const int per = (M + 1023) / 1024;
  const int r0 = tid * per, r1 = min(r0 + per, M);
  int local = 0;
  for (int r = r0; r < r1; ++r) local += flags[r] != 0;
  sums[tid] = local;
  __syncthreads();
  for (int d = 1; d < 1024; d <<= 1) {
    const int v = tid >= d ? sums[tid - d] : 0;
    __syncthreads();
    sums[tid] += v;
    __syncthreads();
  }
  int run = sums[tid] - local;
  for (int r = r0; r < r1; ++r)
    if (flags[r]) list[run++] = r;
  if (tid == 1023) list[M] = sums[1023];
}

// fp32 logits of flagged rows: out[row, v] = sum_k h[row, k] * W[v, k], one FMA
// chain in ascending k per logit (the packed f32x2 FMA below carries two logits of
// two vocabulary entries, each element rounded exactly like a scalar FMA).
// Tile: 64 flagged rows x 128 vocabulary rows per CTA of 4 warps (so that every CTA of
// a 32000-entry vocabulary is resident at once, three per SM). Warp w owns rows
// 16w .. 16w+15: lanes 0-15 rows 16w .. 16w+7, lanes 16-31 rows 16w+8 .. 16w+15; lane
// l owns vocabulary entries 4(l mod 16) .. +3 and 64 + 4(l mod 16) .. +3 (8 x 8
// logits per thread). k is staged KB at a time through two shared-memory buffers (the
// next slab is loaded to registers and stored to the other buffer while this one is
// consumed, one barrier per slab): W transposed to [k][vocab], h as duplicated pairs
// [k][row] (one 16-byte load gives two rows ready for the packed FMA).
constexpr int RB = 64, VB = 128, KB = 16, kRecThreads = 128;

__global__ void __launch_bounds__(kRecThreads, 3) recompute_kernel(const uint16_t* __restrict__ h, int64_t ldh,
                                                                  const uint16_t* __restrict__ W, int64_t V, int K,
                                                                  int M, const int32_t* __restrict__ list,
                                                                  float* __restrict__ out, int skip_upto) {
  pdl_wait();  // inputs written by the previous kernel on the stream are complete from here on
  pdl_trigger();
  __shared__ __align__(16) float2 hs[2][KB][RB];  // (h, h) per row
  __shared__ __align__(16) float ws[2][KB][VB];
  const int count = list[M];
  const int f0 = blockIdx.y * RB;
  if (f0 >= count || count <= skip_upto) return;  // few flagged rows: the streaming kernel takes them
  const int64_t v0 = (int64_t)blockIdx.x * VB;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rbase = warp * 16 + (lane >> 4) * 8;  // first of this thread's 8 rows
  const int vl = (lane & 15) * 4;                  // first of this thread's vocabulary entries (and vl + 64)
  float2 acc[8][4];  // [row][vocab pair]
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = make_float2(0.f, 0.f);

  // staging of one slab: W 128 vocab x 16 k = 256 vectors of 8 (vocab = e / 2, k-half = e % 2, so a
  // vocabulary row's 32 bytes are read by adjacent threads); h 64 rows x 16 k = 128 vectors of 8
  const int hrow = tid >> 1, hk = tid & 1;
  const bool hload = f0 + hrow < count;
  const uint16_t* hsrc = h + (int64_t)(hload ? list[f0 + hrow] : 0) * ldh + hk * 8;
  auto load = [&](int k0, uint4& hv, uint4 (&wv)[2]) {
    hv = hload ? __ldg(reinterpret_cast<const uint4*>(hsrc + k0)) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int e = tid + r * kRecThreads;
      const int64_t vv = v0 + (e >> 1);
      wv[r] = vv < V ? __ldg(reinterpret_cast<const uint4*>(W + vv * K + k0 + (e & 1) * 8))
                     : make_uint4(0, 0, 0, 0);
    }
  };
  auto store = [&](int buf, const uint4& hv, const uint4 (&wv)[2]) {
    float f[8];
    unpack8(hv, f);
#pragma unroll
    for (int i = 0; i < 8; ++i) hs[buf][hk * 8 + i][hrow] = make_float2(f[i], f[i]);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int e = tid + r * kRecThreads;
      unpack8(wv[r], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) ws[buf][(e & 1) * 8 + i][e >> 1] = f[i];
    }
  };
  uint4 hv, wv[2];
  load(0, hv, wv);
  store(0, hv, wv);
  __syncthreads();
  int buf = 0;
  for (int k0 = 0; k0 < K; k0 += KB) {
    const bool more = k0 + KB < K;
    if (more) load(k0 + KB, hv, wv);
#pragma unroll
    for (int kk = 0; kk < KB; ++kk) {
      float2 h2[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 t = *reinterpret_cast<const float4*>(&hs[buf][kk][rbase + 2 * i]);
        h2[2 * i] = make_float2(t.x, t.y);
        h2[2 * i + 1] = make_float2(t.z, t.w);
      }
      const float4 wa = *reinterpret_cast<const float4*>(&ws[buf][kk][vl]);
      const float4 wb = *reinterpret_cast<const float4*>(&ws[buf][kk][64 + vl]);
      const float2 w2[4] = {make_float2(wa.x, wa.y), make_float2(wa.z, wa.w), make_float2(wb.x, wb.y),
                            make_float2(wb.z, wb.w)};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = __ffma2_rn(h2[i], w2[j], acc[i][j]);
    }
    // the other buffer was last read in the previous slab, before the barrier that ended it
    if (more) store(buf ^ 1, hv, wv);
    __syncthreads();
    buf ^= 1;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int f = f0 + rbase + i;
    if (f >= count) continue;
    float* dst = out + (int64_t)list[f] * V;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t v = v0 + (j < 2 ? vl + 2 * j : 64 + vl + 2 * (j - 2));
      if (v < V) dst[v] = acc[i][j].x;
      if (v + 1 < V) dst[v + 1] = acc[i][j].y;
    }
  }
}

// The same fp32 logits for batches of at most kStrMaxCount rows and hidden sizes up to
// 4096, with W streamed once per NR flagged rows instead of once per 64-row tile
// (identical FMA chains, so identical bits), and the flagged rows' tokens taken in the
// same kernel. One launch; the on-device count of flagged rows picks the case:
// stream_rows<1> when exactly one row is flagged (the common case of a trained model's
// rare near-tie), stream_rows<8> for two or more.
// Each warp owns 32 consecutive vocabulary entries (lane = entry) and walks K in tiles of
// 64: a tile (32 rows x 128 bytes of W) is copied coalesced (8 lanes per row, cp.async)
// into the warp's ring of shared-memory slots (rows padded to 144 bytes, so each lane's
// 16-byte reads of its own row are conflict-free), three tiles ahead for one flagged row
// and one ahead for groups of 8, and consumed by each lane along its row. The CTA's NR
// current flagged rows of h sit in shared memory as fp32, [k][row], read as broadcasts;
// packed f32x2 FMAs carry two rows each.
constexpr int kStrWarps = 4, kStrThreads = 128, kStrTK = 64, kStrPad = 72, kStrMaxK = 4096;
constexpr int kStrMaxCount = 24;

// Tiles of W each warp has in flight: four for one flagged row (the h block is small,
// so two CTAs per SM still fit), two for groups of 8 rows (their h block is 8x larger).
__host__ __device__ constexpr int stream_ring(int NR) { return NR == 1 ? 4 : 2; }

inline int stream_smem_bytes(int K, int NR) {
  return K * NR * 4 + kStrWarps * stream_ring(NR) * 32 * kStrPad * 2;
}
// dynamic shared memory of recompute_stream_kernel (either case)
inline int stream_smem_bytes(int K) {
  const int a = stream_smem_bytes(K, 1), b = stream_smem_bytes(K, 8);
  return a > b ? a : b;
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// The rows of `list` (count of them, NR at a time): fp32 logits, per-CTA argmax partials,
// and the last CTA's merge into tokens. smem_str: h of NR rows [K][NR], then the warps'
// tile rings.
template <int NR>
__device__ __forceinline__ void stream_rows(const uint16_t* __restrict__ h, int64_t ldh, const uint16_t* __restrict__ W,
                                            int64_t V, int K, float* __restrict__ out,
                                            ArgBest* __restrict__ arg_part, int32_t* __restrict__ tokens,
                                            unsigned int* __restrict__ ticket, uint8_t* smem_str, const int* list,
                                            int count, ArgBest (&warp_arg)[kStrWarps][8], int& last) {
  float* hsm = reinterpret_cast<float*>(smem_str);                               // [K][NR]
  uint16_t* tiles = reinterpret_cast<uint16_t*>(smem_str + (size_t)K * NR * 4);  // [warp][ring][32][72]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int RING = stream_ring(NR);
  const int64_t vbase = ((int64_t)blockIdx.x * kStrWarps + warp) * 32;
  const int64_t v = vbase + lane;
  uint16_t* ring = tiles + warp * RING * 32 * kStrPad;  // this warp's RING tile slots
  const int ntile = K / kStrTK;
  // tile t into slot t mod RING: copy q moves rows 4q .. 4q+3, lane l the 16 bytes
  // (l mod 8) of row 4q + l/8 (coalesced); rows past V are zero-filled. One commit group
  // per tile (an empty group past the last tile keeps the wait count uniform).
  auto load_tile = [&](int t) {
    if (t < ntile) {
      uint16_t* slot = ring + (t % RING) * 32 * kStrPad;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int row = q * 4 + (lane >> 3);
        const int64_t vv = vbase + row;
        uint16_t* dst = slot + row * kStrPad + (lane & 7) * 8;
        if (vv < V)
          cp_async16(dst, W + vv * K + t * kStrTK + (lane & 7) * 8);
        else
          *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
      }
    }
    cp_async_commit();
  };
  for (int r0 = 0; r0 < count; r0 += NR) {
    const int nr = min(NR, count - r0);
    __syncthreads();  // the previous rows of h and the previous partials are no longer read
    for (int e = threadIdx.x; e < NR * (K / 8); e += kStrThreads) {
      const int r = e % NR, kv = e / NR;
      float f[8];
      if (r < nr) {
        unpack8(__ldg(reinterpret_cast<const uint4*>(h + (int64_t)list[r0 + r] * ldh) + kv), f);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) hsm[(kv * 8 + i) * NR + r] = f[i];
    }
    __syncthreads();
    float acc[NR];
#pragma unroll
    for (int j = 0; j < NR; ++j) acc[j] = 0.f;
    // RING - 1 tiles in flight ahead of the one being consumed, copied straight into
    // the warp's shared-memory slots
    __syncwarp();  // the slots' previous contents (earlier rows) are no longer read
#pragma unroll
    for (int t = 0; t < RING - 1; ++t) load_tile(t);
    auto step = [&](int t) {
      load_tile(t + RING - 1);       // into the slot consumed at step t - 1
      cp_async_wait<RING - 1>();     // this lane's copies of tile t have landed
      __syncwarp();                  // and every lane's
      const uint16_t* my = ring + (t % RING) * 32 * kStrPad;
#pragma unroll
      for (int c = 0; c < kStrTK / 8; ++c) {
        float w[8];
        unpack8(*reinterpret_cast<const uint4*>(my + lane * kStrPad + c * 8), w);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float* hk = hsm + (t * kStrTK + c * 8 + i) * NR;
          if constexpr (NR == 1) {
            acc[0] = __fmaf_rn(hk[0], w[i], acc[0]);
          } else {
            // packed pairs of rows; each element rounds exactly like a scalar FMA
#pragma unroll
            for (int j = 0; j < NR; j += 4) {
              const float4 a = *reinterpret_cast<const float4*>(hk + j);
              const float2 ww = make_float2(w[i], w[i]);
              const float2 p0 = __ffma2_rn(make_float2(a.x, a.y), ww, make_float2(acc[j], acc[j + 1]));
              const float2 p1 = __ffma2_rn(make_float2(a.z, a.w), ww, make_float2(acc[j + 2], acc[j + 3]));
              acc[j] = p0.x;
              acc[j + 1] = p0.y;
              acc[j + 2] = p1.x;
              acc[j + 3] = p1.y;
            }
          }
        }
      }
    };
    for (int t = 0; t < ntile; ++t) {
      step(t);
      __syncwarp();  // every lane is done with slot t mod RING before it is refilled
    }
    cp_async_wait<0>();
    // fp32 logits out, and this CTA's argmax of each row over its 128 entries (lowest
    // index on ties, NaN never wins): lanes by an xor tree, then the warps in order
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      if (r < nr && v < V) out[(int64_t)list[r0 + r] * V + v] = acc[r];
      ArgBest b{v < V ? sanitize(acc[r]) : -INFINITY, v < V ? (int)v : 0x7FFFFFFF};
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        const float ov = __shfl_xor_sync(kFullMask, b.v, o);
        const int oi = __shfl_xor_sync(kFullMask, b.i, o);
        if (better(ov, oi, b.v, b.i)) b = ArgBest{ov, oi};
      }
      if (lane == 0) warp_arg[warp][r] = b;
    }
    __syncthreads();
    if (threadIdx.x < nr) {
      ArgBest b = warp_arg[0][threadIdx.x];
      for (int w2 = 1; w2 < kStrWarps; ++w2)
        if (better(warp_arg[w2][threadIdx.x].v, warp_arg[w2][threadIdx.x].i, b.v, b.i)) b = warp_arg[w2][threadIdx.x];
      arg_part[(int64_t)(r0 + threadIdx.x) * gridDim.x + blockIdx.x] = b;
    }
  }
  // the CTA that finishes last (an integer ticket zeroed by top2_kernel; it orders no
  // value) merges the CTAs' partials in CTA order and writes the tokens
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    last = atomicAdd(ticket, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  // per flagged row: thread t takes partials t, t + 128, ... (read from L2, where the
  // other CTAs' writes are), then an xor tree over the lanes and the warps in order
  for (int f = 0; f < count; ++f) {
    const ArgBest* p = arg_part + (int64_t)f * gridDim.x;
    ArgBest b{-INFINITY, 0x7FFFFFFF};
    for (unsigned c = threadIdx.x; c < gridDim.x; c += kStrThreads) {
      const float cv = __ldcg(&p[c].v);
      const int ci = __ldcg(&p[c].i);
      if (better(cv, ci, b.v, b.i)) b = ArgBest{cv, ci};
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const float ov = __shfl_xor_sync(kFullMask, b.v, o);
      const int oi = __shfl_xor_sync(kFullMask, b.i, o);
      if (better(ov, oi, b.v, b.i)) b = ArgBest{ov, oi};
    }
    __syncthreads();  // warp_arg of the previous row is read
    if (lane == 0) warp_arg[warp][0] = b;
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int w2 = 1; w2 < kStrWarps; ++w2)
        if (better(warp_arg[w2][0].v, warp_arg[w2][0].i, b.v, b.i)) b = warp_arg[w2][0];
      tokens[list[f]] = b.i;
    }
  }
}

// Both streaming cases in one launch: the flagged rows are listed with one ballot (M <=
// kStrMaxCount), then exactly one flagged row reads W once with one fp32 chain per lane
// (stream_rows<1>), two or more read it once per group of 8 (stream_rows<8>), and no
// flagged row returns at once.
__global__ void __launch_bounds__(kStrThreads) recompute_stream_kernel(const uint16_t* __restrict__ h, int64_t ldh,
                                                                      const uint16_t* __restrict__ W, int64_t V,
                                                                      int K, int M, const int32_t* __restrict__ flags,
                                                                      float* __restrict__ out,
                                                                      ArgBest* __restrict__ arg_part,
                                                                      int32_t* __restrict__ tokens,
                                                                      unsigned int* __restrict__ ticket) {
  pdl_wait();  // inputs written by the previous kernel on the stream are complete from here on
  pdl_trigger();
  extern __shared__ __align__(16) uint8_t smem_str[];
  __shared__ int list[kStrMaxCount + 1];  // flagged rows, ascending (M <= kStrMaxCount)
  __shared__ ArgBest warp_arg[kStrWarps][8];
  __shared__ int last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {  // the flagged rows in order: one ballot over M <= 24 rows
    const bool f = lane < M && flags[lane] != 0;
    const unsigned mask = __ballot_sync(kFullMask, f);
    if (f) list[__popc(mask & ((1u << lane) - 1u))] = lane;
    if (lane == 0) list[kStrMaxCount] = __popc(mask);
  }
  __syncthreads();
  const int count = list[kStrMaxCount];
  if (count == 1)
    stream_rows<1>(h, ldh, W, V, K, out, arg_part, tokens, ticket, smem_str, list, count, warp_arg, last);
  else if (count >= 2)
    stream_rows<8>(h, ldh, W, V, K, out, arg_part, tokens, ticket, smem_str, list, count, warp_arg, last);
}

// Token of each flagged row = argmax of its fp32 logits (lowest index on ties), a cluster
// of kParts CTAs per row as in top2_kernel (the argmax is exact, so the split does not
// change it).
__global__ void __cluster_dims__(kParts, 1, 1) __launch_bounds__(kThreads)
    argmax_kernel(const float* __restrict__ logits, int64_t V, const int32_t* __restrict__ flags,
                  int32_t* __restrict__ tokens) {
  pdl_wait();  // inputs written by the previous kernel on the stream are complete from here on
  pdl_trigger();
  __shared__ float wv[kThreads / 32];
  __shared__ int wi[kThreads / 32];
  __shared__ float part_v;
  __shared__ int part_i;
  const int64_t row = blockIdx.x / kParts;
  if (!flags[row]) return;  // the same for every CTA of the cluster
  const uint32_t part = cluster_rank();
  const float* src = logits + row * V;
  const int64_t per = (V + kParts - 1) / kParts;
  const int64_t j0 = (int64_t)part * per, j1 = min(V, j0 + per);
  float best = -INFINITY;
  int bi_ = 0x7FFFFFFF;
  for (int64_t j = j0 + threadIdx.x; j < j1; j += kThreads) {
    const float v = sanitize(src[j]);
    if (better(v, (int)j, best, bi_)) {
      best = v;
      bi_ = (int)j;
    }
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const float v = __shfl_xor_sync(kFullMask, best, o);
    const int i = __shfl_xor_sync(kFullMask, bi_, o);
    if (better(v, i, best, bi_)) {
      best = v;
      bi_ = i;
    }
  }
  if ((threadIdx.x & 31) == 0) {
    wv[threadIdx.x >> 5] = best;
    wi[threadIdx.x >> 5] = bi_;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = wv[0];
    int bi2 = wi[0];
    for (int w = 1; w < kThreads / 32; ++w)
      if (better(wv[w], wi[w], b, bi2)) {
        b = wv[w];
        bi2 = wi[w];
      }
    part_v = b;
    part_i = bi2;
  }
  cluster_barrier();
  if (part == 0 && threadIdx.x == 0) {
    float b = part_v;
    int bi2 = part_i;
    for (uint32_t p = 1; p < kParts; ++p) {
      const float v = ld_cluster_f32(map_to_rank(smem_u32(&part_v), p));
      const int i = ld_cluster_s32(map_to_rank(smem_u32(&part_i), p));
      if (better(v, i, b, bi2)) {
        b = v;
        bi2 = i;
      }
    }
    tokens[row] = bi2;
  }
  cluster_barrier();
}

}  // namespace lmhead
}  // namespace bi
