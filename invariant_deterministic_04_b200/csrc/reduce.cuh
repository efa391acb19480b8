// Row reductions over the vocabulary or feature axis, and temperature sampling,
// one row per CTA.
//
// Source: "Defeating Nondeterminism in LLM Inference" technical summary
// (mobiles-han blog), section 他の演算子 (RMSNorm, MatMul, mean/reduction etc.):
// log_softmax and mean join the operations given batch-invariant kernels, and a
// mean is reduced in one fixed order (no split, or only a split of fixed size).
// Why the log-probability and the sampled token must not move with the batch:
// Techzine, "Thinking Machines wil AI voorspelbaarder maken" (sampling and
// training bit-identical, hence on-policy RL), and the French "température zéro"
// blog, section "Le mensonge de la température zéro".
//
// Reduction order of a row (a function of the row length N only):
//   thread t (of 256) owns the 8-element vectors t, t+256, t+512, ... and folds
//   their elements in order (vector by vector, element 0..7) into one fp32 value;
//   the 32 lane values of a warp are combined by an xor-butterfly (16, 8, 4, 2, 1);
//   the 8 warp values are combined as (((w0 + w1) + w2) + ...) + w7.
// Rows of up to 32768 elements stay in registers (read from HBM once); longer rows
// are re-read for each pass (from L2) in the same order.
// Max and argmax are exact, so their combination order does not matter; argmax
// takes the lowest index among equal values.
#pragma once

#include "device.cuh"

namespace bi {
namespace red {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr float kLog2e = 1.4426950408889634f;

// block-wide fixed-order fp32 sum (all threads get the result)
__device__ __forceinline__ float block_sum(float v, float* sh) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v = __fadd_rn(v, __shfl_xor_sync(kFullMask, v, off));
  __syncthreads();  // sh may still be read from a previous reduction
  if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = v;
  __syncthreads();
  float t = sh[0];
#pragma unroll
  for (int i = 1; i < kWarps; ++i) t = __fadd_rn(t, sh[i]);
  return t;
}

__device__ __forceinline__ float block_max(float v, float* sh) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v = fmaxf(v, __shfl_xor_sync(kFullMask, v, off));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = v;
  __syncthreads();
  float t = sh[0];
#pragma unroll
  for (int i = 1; i < kWarps; ++i) t = fmaxf(t, sh[i]);
  return t;
}

// exp(x - m) as 2^(x log2 e - m log2 e): one FMA (mc = m * log2 e rounded once) and
// the SFU exp2; x == -inf gives 0
__device__ __forceinline__ float exp_shifted(float x, float mc) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(__fmaf_rn(x, kLog2e, -mc)));
  return y;
}

// The row's vectors: in registers (NV > 0, N <= NV * 256 * 8) or re-read (NV == 0).
template <int NV>
struct Row {
  uint4 v[NV > 0 ? NV : 1];
  const uint4* src;
  int nvec;
  __device__ __forceinline__ void load(const uint16_t* row, int N) {
    src = reinterpret_cast<const uint4*>(row);
    nvec = N >> 3;
    if (NV > 0) {
#pragma unroll
      for (int j = 0; j < NV; ++j) {
        const int idx = threadIdx.x + j * kThreads;
        if (idx < nvec) v[j] = __ldcs(src + idx);
      }
    }
  }
  // f(vector index, 8 floats) over this thread's vectors, in ascending order
  template <class F>
  __device__ __forceinline__ void each(F&& f) const {
    if (NV > 0) {
#pragma unroll
      for (int j = 0; j < NV; ++j) {
        const int idx = threadIdx.x + j * kThreads;
        if (idx < nvec) {
          float e[8];
          unpack8(v[j], e);
          f(idx, e);
        }
      }
    } else {
      for (int idx = threadIdx.x; idx < nvec; idx += kThreads) {
        float e[8];
        unpack8(__ldg(src + idx), e);
        f(idx, e);
      }
    }
  }
};

// max and log(sum exp(x - max)) of a row: lse = max + log(sum)
template <int NV>
__device__ __forceinline__ float row_lse(const Row<NV>& row, float* sh) {
  float m = -INFINITY;
  row.each([&](int, const float(&e)[8]) {
#pragma unroll
    for (int k = 0; k < 8; ++k) m = fmaxf(m, e[k]);
  });
  m = block_max(m, sh);
  const float mc = __fmul_rn(m, kLog2e);
  float s = 0.f;
  row.each([&](int, const float(&e)[8]) {
#pragma unroll
    for (int k = 0; k < 8; ++k) s = __fadd_rn(s, exp_shifted(e[k], mc));
  });
  s = block_sum(s, sh);
  return __fadd_rn(m, logf(s));
}

template <int NV>
__global__ void __launch_bounds__(kThreads) log_softmax_kernel(const uint16_t* __restrict__ x, int64_t ldx,
                                                               float* __restrict__ y, int64_t ldy, int N) {
  __shared__ float sh[kWarps];
  Row<NV> row;
  row.load(x + (int64_t)blockIdx.x * ldx, N);
  const float lse = row_lse(row, sh);
  float4* yr = reinterpret_cast<float4*>(y + (int64_t)blockIdx.x * ldy);
  row.each([&](int idx, const float(&e)[8]) {
    __stcs(yr + 2 * idx, make_float4(__fsub_rn(e[0], lse), __fsub_rn(e[1], lse), __fsub_rn(e[2], lse),
                                     __fsub_rn(e[3], lse)));
    __stcs(yr + 2 * idx + 1, make_float4(__fsub_rn(e[4], lse), __fsub_rn(e[5], lse), __fsub_rn(e[6], lse),
                                         __fsub_rn(e[7], lse)));
  });
}

template <int NV>
__global__ void __launch_bounds__(kThreads) token_logprob_kernel(const uint16_t* __restrict__ x, int64_t ldx,
                                                                 const int32_t* __restrict__ tokens,
                                                                 float* __restrict__ out, int N) {
  __shared__ float sh[kWarps];
  Row<NV> row;
  const uint16_t* xr = x + (int64_t)blockIdx.x * ldx;
  row.load(xr, N);
  const float lse = row_lse(row, sh);
  if (threadIdx.x == 0) {
    const int t = tokens[blockIdx.x];
    if (t < 0 || t >= N) {
      record_error(BI_ERR_DEVICE_INDEX);
      out[blockIdx.x] = __int_as_float(0x7fc00000);
    } else {
      out[blockIdx.x] = __fsub_rn(__uint_as_float((uint32_t)xr[t] << 16), lse);
    }
  }
}

template <int NV>
__global__ void __launch_bounds__(kThreads) row_mean_kernel(const uint16_t* __restrict__ x, int64_t ldx,
                                                            float* __restrict__ y, int K) {
  __shared__ float sh[kWarps];
  Row<NV> row;
  row.load(x + (int64_t)blockIdx.x * ldx, K);
  float s = 0.f;
  row.each([&](int, const float(&e)[8]) {
#pragma unroll
    for (int k = 0; k < 8; ++k) s = __fadd_rn(s, e[k]);
  });
  s = block_sum(s, sh);
  if (threadIdx.x == 0) y[blockIdx.x] = __fdiv_rn(s, (float)K);
}

// ---------------------------------------------------------------------------
// Philox4x64-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as
// 1, 2, 3", SC 2011): ten rounds over a 256-bit counter under a 128-bit key.
// Round: (x0, x1, x2, x3) -> (hi(M1 x2) ^ x1 ^ k0, lo(M1 x2), hi(M0 x0) ^ x3 ^ k1,
// lo(M0 x0)), then the key takes a Weyl step.

struct U64x4 {
  uint64_t w[4];
};

__device__ __forceinline__ U64x4 philox4x64_10(uint64_t c0, uint64_t c1, uint64_t c2, uint64_t c3, uint64_t k0,
                                               uint64_t k1) {
  constexpr uint64_t M0 = 0xD2E7470EE14C6C93ull, M1 = 0xCA5A826395121157ull;
  constexpr uint64_t W0 = 0x9E3779B97F4A7C15ull, W1 = 0xBB67AE8584CAA73Bull;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t hi0 = __umul64hi(M0, c0), lo0 = M0 * c0;
    const uint64_t hi1 = __umul64hi(M1, c2), lo1 = M1 * c2;
    c0 = hi1 ^ c1 ^ k0;
    c1 = lo1;
    c2 = hi0 ^ c3 ^ k1;
    c3 = lo0;
    k0 += W0;
    k1 += W1;
  }
  return U64x4{{c0, c1, c2, c3}};
}

// u in (0, 1): (top 23 bits of a 32-bit half + 1/2) * 2^-23, exact in fp32
__device__ __forceinline__ float half_to_uniform(uint32_t h) {
  return __fmul_rn(__fadd_rn((float)(h >> 9), 0.5f), 1.1920928955078125e-07f);
}

// The uniforms of vocabulary entries 8 idx .. 8 idx + 7 of a row: one Philox block,
// counter (idx, step), key (seed, 0); entry 8 idx + k takes word k / 2, its low half
// for even k and its high half for odd k.
__device__ __forceinline__ void uniforms8(uint64_t seed, uint64_t step, int idx, float (&u)[8]) {
  const U64x4 r = philox4x64_10((uint64_t)idx, step, 0ull, 0ull, seed, 0ull);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    u[2 * k] = half_to_uniform((uint32_t)r.w[k]);
    u[2 * k + 1] = half_to_uniform((uint32_t)(r.w[k] >> 32));
  }
}

__global__ void __launch_bounds__(kThreads) uniforms_kernel(const uint64_t* __restrict__ seeds,
                                                            const uint64_t* __restrict__ steps, float* __restrict__ u,
                                                            int64_t ldu, int V) {
  const uint64_t seed = seeds[blockIdx.x], step = steps[blockIdx.x];
  float4* ur = reinterpret_cast<float4*>(u + (int64_t)blockIdx.x * ldu);
  for (int idx = threadIdx.x; idx < (V >> 3); idx += kThreads) {
    float v[8];
    uniforms8(seed, step, idx, v);
    ur[2 * idx] = make_float4(v[0], v[1], v[2], v[3]);
    ur[2 * idx + 1] = make_float4(v[4], v[5], v[6], v[7]);
  }
}

// (value, index) pair order for argmax: larger value, then lower index
__device__ __forceinline__ bool better(float v, int i, float bv, int bi_) { return v > bv || (v == bv && i < bi_); }

// Temperature sampling by the Gumbel-max rule: token = argmax_i (x_i / T + g_i) with
// g_i = -log(-log u_i), score = fma(x_i, 1/T, g_i) in fp32 (1/T rounded once). The
// inner log is the accurate logf (for u near 1, -log u is tiny and its relative
// error would pass straight into g); the outer one is the SFU log2 times ln 2, whose
// absolute error (~1e-7) is what g sees.
// A row is split over a cluster of kSampleParts CTAs, part p taking vectors
// p * ceil(n/8) .. of the row's n 8-element vectors (a split fixed by V alone); the
// parts' (score, index) maxima meet in CTA 0 through distributed shared memory. An
// argmax is exact, so the split does not change the result.
constexpr int kSampleParts = 8;

__global__ void __cluster_dims__(kSampleParts, 1, 1) __launch_bounds__(kThreads)
    sample_kernel(const uint16_t* __restrict__ x, int64_t ldx, const uint64_t* __restrict__ seeds,
                  const uint64_t* __restrict__ steps, float inv_t, int32_t* __restrict__ tokens, int V) {
  __shared__ float shv[kWarps];
  __shared__ int shi[kWarps];
  __shared__ float part_v;
  __shared__ int part_i;
  const int row = blockIdx.x / kSampleParts;
  const uint32_t part = cluster_rank();
  const int nvec = V >> 3, per = (nvec + kSampleParts - 1) / kSampleParts;
  const int v0 = (int)part * per, v1 = min(nvec, v0 + per);
  const uint4* xr = reinterpret_cast<const uint4*>(x + (int64_t)row * ldx);
  const uint64_t seed = seeds[row], step = steps[row];
  float bv = -INFINITY;
  int bidx = INT_MAX;
  for (int idx = v0 + (int)threadIdx.x; idx < v1; idx += kThreads) {
    float e[8], u[8];
    unpack8(__ldcs(xr + idx), e);
    uniforms8(seed, step, idx, u);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float g = -__logf(-logf(u[k]));
      const float sc = __fmaf_rn(e[k], inv_t, g);
      if (better(sc, 8 * idx + k, bv, bidx)) {
        bv = sc;
        bidx = 8 * idx + k;
      }
    }
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const float ov = __shfl_xor_sync(kFullMask, bv, off);
    const int oi = __shfl_xor_sync(kFullMask, bidx, off);
    if (better(ov, oi, bv, bidx)) {
      bv = ov;
      bidx = oi;
    }
  }
  if ((threadIdx.x & 31) == 0) {
    shv[threadIdx.x >> 5] = bv;
    shi[threadIdx.x >> 5] = bidx;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float v = shv[0];
    int i = shi[0];
    for (int w = 1; w < kWarps; ++w)
      if (better(shv[w], shi[w], v, i)) {
        v = shv[w];
        i = shi[w];
      }
    part_v = v;
    part_i = i;
  }
  cluster_barrier();  // every part's maximum is in its shared memory
  if (part == 0 && threadIdx.x == 0) {
    float v = part_v;
    int i = part_i;
    for (uint32_t p = 1; p < kSampleParts; ++p) {
      const float pv = ld_cluster_f32(map_to_rank(smem_u32(&part_v), p));
      const int pi = ld_cluster_s32(map_to_rank(smem_u32(&part_i), p));
      if (better(pv, pi, v, i)) {
        v = pv;
        i = pi;
      }
    }
    // a row whose scores are all NaN (NaN logits) has no maximum: report index 0 and the error
    if (i == INT_MAX) {
      record_error(BI_ERR_DEVICE_INDEX);
      i = 0;
    }
    tokens[row] = i;
  }
  cluster_barrier();  // no part leaves while part 0 may still read its shared memory
}

// vectors per thread of the register-resident variant for a row of N elements, or 0
// (re-read) above 32768
inline int vectors_per_thread(int64_t N) {
  const int64_t per = (N / 8 + kThreads - 1) / kThreads;
  return per <= 1 ? 1 : per <= 2 ? 2 : per <= 4 ? 4 : per <= 8 ? 8 : per <= 16 ? 16 : 0;
}

// launch kernel template KER<NV> with the variant that fits N
#define BI_RED_DISPATCH(KER, N, GRID, ST, ...)                                                 \
  do {                                                                                       \
    switch (::bi::red::vectors_per_thread(N)) {                                              \
      case 1: KER<1><<<(GRID), ::bi::red::kThreads, 0, (ST)>>>(__VA_ARGS__); break;           \
      case 2: KER<2><<<(GRID), ::bi::red::kThreads, 0, (ST)>>>(__VA_ARGS__); break;           \
      case 4: KER<4><<<(GRID), ::bi::red::kThreads, 0, (ST)>>>(__VA_ARGS__); break;           \
      case 8: KER<8><<<(GRID), ::bi::red::kThreads, 0, (ST)>>>(__VA_ARGS__); break;           \
      case 16: KER<16><<<(GRID), ::bi::red::kThreads, 0, (ST)>>>(__VA_ARGS__); break;         \
      default: KER<0><<<(GRID), ::bi::red::kThreads, 0, (ST)>>>(__VA_ARGS__); break;          \
    }                                                                                        \
  } while (0)

}  // namespace red
}  // namespace bi
