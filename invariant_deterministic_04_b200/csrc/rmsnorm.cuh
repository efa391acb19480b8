// RMSNorm: each row reduced by one CTA, rows dealt to a persistent grid.
//
// Source: "Defeating Nondeterminism in LLM Inference" technical summary
// (mobiles-han blog), section 対応策：バッチ不変なカーネル設計, kernel table, row
// RMSNorm: keep the data-parallel strategy (each row reduced by itself) at every
// batch size instead of switching to a split reduction when the batch is small.
//
// Reduction order of a row (a function of K only):
//   thread t (of 128) owns the 16-byte vectors t, t+128, t+256, ... of the row and
//   accumulates their 8 squares each, in order, with one fp32 FMA chain;
//   the 32 lane sums of a warp are added by an xor-butterfly (offsets 16, 8, 4, 2, 1);
//   the 4 warp sums are added as ((w0 + w1) + w2) + w3.
// Then y = bf16_rne((x * rstd) * w) with rstd = rsqrt(sum / K + eps).
// Each row is read from HBM once (kept in registers) and written once, after the
// whole row has been read, so y may alias x.
//
// Scheduling (no effect on any row's arithmetic): CTA b takes rows b, b + grid,
// b + 2 grid, ...; while it reduces and writes one row, the loads of its next row
// are already in flight, so reads and writes of different rows overlap in HBM
// instead of the whole batch reading first and writing after. Batches of more than
// four waves of resident CTAs get one CTA per row instead.
#pragma once

#include "device.cuh"

namespace bi {
namespace rms {

constexpr int kThreads = 128;

template <int NV>  // 16-byte vectors per thread
__device__ __forceinline__ void load_row(const uint4* xr, int nvec, uint4 (&v)[NV]) {
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int idx = threadIdx.x + j * kThreads;
    if (idx < nvec) v[j] = __ldcs(xr + idx);
  }
}

template <int NV>  // 16-byte vectors per thread
__global__ void __launch_bounds__(kThreads) rmsnorm_kernel(const uint16_t* x,
                                                           int64_t ldx,
                                                           const uint16_t* __restrict__ w,
                                                           uint16_t* y, int64_t ldy,
                                                           int64_t M, int K, float eps) {
  __shared__ float warp_sum[2][kThreads / 32];
  const int nvec = K >> 3;
  const uint4* wr = reinterpret_cast<const uint4*>(w);
  int64_t row = blockIdx.x;
  uint4 v[NV], vn[NV];
  pdl_wait();  // the previous kernel on the stream has written x (or still reads y) until now
  pdl_trigger();
  load_row<NV>(reinterpret_cast<const uint4*>(x + row * ldx), nvec, v);
  for (int it = 0; row < M; row += gridDim.x, ++it) {
    const int64_t next = row + gridDim.x;
    if (next < M) load_row<NV>(reinterpret_cast<const uint4*>(x + next * ldx), nvec, vn);
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int idx = threadIdx.x + j * kThreads;
      if (idx < nvec) {
        float f[8];
        unpack8(v[j], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = __fmaf_rn(f[e], f[e], ss);
      }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(kFullMask, ss, off));
    // two slots: a warp that runs ahead writes the other one (the slot it reuses two
    // rows later is free, every thread having passed the barrier in between)
    float* ws = warp_sum[it & 1];
    if ((threadIdx.x & 31) == 0) ws[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = ws[0];
#pragma unroll
    for (int i = 1; i < kThreads / 32; ++i) tot = __fadd_rn(tot, ws[i]);
    const float rstd = rsqrtf(__fadd_rn(__fdiv_rn(tot, (float)K), eps));

    uint4* yr = reinterpret_cast<uint4*>(y + row * ldy);
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int idx = threadIdx.x + j * kThreads;
      if (idx < nvec) {
        float f[8], g[8];
        unpack8(v[j], f);
        unpack8(__ldg(wr + idx), g);
        uint4 o;
        o.x = pack_bf16x2(__fmul_rn(__fmul_rn(f[0], rstd), g[0]), __fmul_rn(__fmul_rn(f[1], rstd), g[1]));
        o.y = pack_bf16x2(__fmul_rn(__fmul_rn(f[2], rstd), g[2]), __fmul_rn(__fmul_rn(f[3], rstd), g[3]));
        o.z = pack_bf16x2(__fmul_rn(__fmul_rn(f[4], rstd), g[4]), __fmul_rn(__fmul_rn(f[5], rstd), g[5]));
        o.w = pack_bf16x2(__fmul_rn(__fmul_rn(f[6], rstd), g[6]), __fmul_rn(__fmul_rn(f[7], rstd), g[7]));
        yr[idx] = o;
      }
    }
#pragma unroll
    for (int j = 0; j < NV; ++j) v[j] = vn[j];
  }
}

// Resident CTAs per SM for the persistent grid (registers of the row and of the
// prefetched next row bound it at large K).
template <int NV>
constexpr int ctas_per_sm() {
  return NV <= 4 ? 8 : NV <= 8 ? 4 : 2;
}

template <int NV>
inline cudaError_t launch_nv(const uint16_t* x, int64_t ldx, const uint16_t* w, uint16_t* y, int64_t ldy, int64_t M,
                             int K, float eps, int sms, cudaStream_t st) {
  // up to 4 waves of resident CTAs: the persistent grid (each CTA overlaps its next
  // row's loads with the current row's stores); beyond that one CTA per row, which
  // the hardware schedules as CTAs retire (measured faster at M = 65536)
  const int64_t cap = (int64_t)sms * ctas_per_sm<NV>();
  const unsigned grid = (unsigned)(M <= 4 * cap ? (M < cap ? M : cap) : M);
  return launch_pdl(rmsnorm_kernel<NV>, dim3(grid), dim3(kThreads), 0, st, x, ldx, w, y, ldy, M, K, eps);
}

inline cudaError_t launch(const uint16_t* x, int64_t ldx, const uint16_t* w, uint16_t* y,
                          int64_t ldy, int64_t M, int K, float eps, int sms, cudaStream_t st) {
  const int nvec = K / 8;
  const int per = (nvec + kThreads - 1) / kThreads;
  if (per <= 1) return launch_nv<1>(x, ldx, w, y, ldy, M, K, eps, sms, st);
  if (per <= 2) return launch_nv<2>(x, ldx, w, y, ldy, M, K, eps, sms, st);
  if (per <= 4) return launch_nv<4>(x, ldx, w, y, ldy, M, K, eps, sms, st);
  if (per <= 8) return launch_nv<8>(x, ldx, w, y, ldy, M, K, eps, sms, st);
  return launch_nv<16>(x, ldx, w, y, ldy, M, K, eps, sms, st);
}

}  // namespace rms
}  // namespace bi
