// Row-wise glue of a Llama-style decoder step: row gather (embedding lookup,
// row selection), rotary position embedding, SwiGLU and the residual add.
//
// Each is elementwise or a copy: an output element depends only on the same
// row's inputs, so these are batch-invariant by construction (no reductions).
// They exist so that a whole decoder step runs in this library's kernels
// between the batch-invariant reductions (RMSNorm, matmul, attention, LM head)
// of the "Defeating Nondeterminism in LLM Inference" summary's kernel table.
#pragma once

#include "device.cuh"

namespace bi {
namespace glue {

// dst[m, :] = src[idx[m], :] (width bf16 per row); one warp per row, 16-byte copies.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* __restrict__ src, int64_t ld_src,
                                                          int64_t nrows_src, const int32_t* __restrict__ idx,
                                                          int M, int64_t width, uint16_t* __restrict__ dst,
                                                          int64_t ld_dst) {
  pdl_wait();  // inputs written by the previous kernel on the stream are complete from here on
  pdl_trigger();
  const int64_t m = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (m >= M) return;
  const int64_t r = idx[m];
  uint4* d = reinterpret_cast<uint4*>(dst + m * ld_dst);
  if (r < 0 || r >= nrows_src) {
    if (lane == 0) record_error(BI_ERR_DEVICE_INDEX);
    for (int64_t i = lane; i < width / 8; i += 32) d[i] = make_uint4(0, 0, 0, 0);
    return;
  }
  const uint4* s = reinterpret_cast<const uint4*>(src + r * ld_src);
  for (int64_t i = lane; i < width / 8; i += 32) d[i] = __ldg(s + i);
}

// Rotary embedding, rotate-half form, in place on x[t, h*D .. h*D + D) (row stride
// ldx): for i < D/2, with (c, s) = table[pos[t] * D/2 + i],
//   x[i]       <- x[i] * c - x[i + D/2] * s
//   x[i + D/2] <- x[i + D/2] * c + x[i] * s
// in fp32 as fma(a, c, -(b * s)) and fma(b, c, a * s), rounded to bf16.
// One thread per (token, head, i).
__global__ void __launch_bounds__(256) rope_kernel(uint16_t* __restrict__ x, int64_t ldx, int T, int H, int D,
                                                   const int32_t* __restrict__ pos, const float2* __restrict__ table,
                                                   int max_pos) {
  pdl_wait();  // inputs written by the previous kernel on the stream are complete from here on
  pdl_trigger();
  const int half = D / 2;
  const int64_t e = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (e >= (int64_t)T * H * half) return;
  const int i = (int)(e % half);
  const int64_t th = e / half;
  const int h = (int)(th % H);
  const int t = (int)(th / H);
  const int p = pos[t];
  if (p < 0 || p >= max_pos) {
    if (i == 0) record_error(BI_ERR_DEVICE_INDEX);
    return;
  }
  uint16_t* row = x + (int64_t)t * ldx + (int64_t)h * D;
  const float a = __uint_as_float((uint32_t)row[i] << 16);
  const float b = __uint_as_float((uint32_t)row[i + half] << 16);
  const float2 cs = table[(int64_t)p * half + i];
  const float y1 = __fmaf_rn(a, cs.x, -__fmul_rn(b, cs.y));
  const float y2 = __fmaf_rn(b, cs.x, __fmul_rn(a, cs.y));
  row[i] = to_bf16_bits(y1);
  row[i + half] = to_bf16_bits(y2);
}

// out[m, j] = bf16( silu(g) * u ), g = gu[m, j], u = gu[m, F + j],
// silu(g) = g / (1 + exp(-g)) in fp32 (expf, then an IEEE division).
__global__ void __launch_bounds__(256) swiglu_kernel(const uint16_t* __restrict__ gu, int64_t ld_gu,
                                                     uint16_t* __restrict__ out, int64_t ld_out, int M, int F) {
  pdl_wait();  // inputs written by the previous kernel on the stream are complete from here on
  pdl_trigger();
  const int64_t e = (int64_t)blockIdx.x * 256 + threadIdx.x;  // one thread per 8 outputs
  const int64_t per_row = F / 8;
  if (e >= (int64_t)M * per_row) return;
  const int64_t m = e / per_row;
  const int64_t j = (e % per_row) * 8;
  float g[8], u[8];
  unpack8(__ldg(reinterpret_cast<const uint4*>(gu + m * ld_gu + j)), g);
  unpack8(__ldg(reinterpret_cast<const uint4*>(gu + m * ld_gu + F + j)), u);
  float y[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float s = __fdiv_rn(g[k], __fadd_rn(1.f, expf(-g[k])));
    y[k] = __fmul_rn(s, u[k]);
  }
  uint4 o;
  o.x = pack_bf16x2(y[0], y[1]);
  o.y = pack_bf16x2(y[2], y[3]);
  o.z = pack_bf16x2(y[4], y[5]);
  o.w = pack_bf16x2(y[6], y[7]);
  *reinterpret_cast<uint4*>(out + m * ld_out + j) = o;
}

// out = bf16(a + b) elementwise (fp32 add of the two bf16 values), n % 8 == 0.
// out may alias a or b (each thread reads its 8 elements before writing them).
__global__ void __launch_bounds__(256) add_kernel(const uint16_t* a, const uint16_t* b, uint16_t* out, int64_t n) {
  pdl_wait();  // inputs written by the previous kernel on the stream are complete from here on
  pdl_trigger();
  const int64_t e = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (e >= n / 8) return;
  float x[8], y[8];
  unpack8(reinterpret_cast<const uint4*>(a)[e], x);
  unpack8(reinterpret_cast<const uint4*>(b)[e], y);
  uint4 o;
  o.x = pack_bf16x2(__fadd_rn(x[0], y[0]), __fadd_rn(x[1], y[1]));
  o.y = pack_bf16x2(__fadd_rn(x[2], y[2]), __fadd_rn(x[3], y[3]));
  o.z = pack_bf16x2(__fadd_rn(x[4], y[4]), __fadd_rn(x[5], y[5]));
  o.w = pack_bf16x2(__fadd_rn(x[6], y[6]), __fadd_rn(x[7], y[7]));
  reinterpret_cast<uint4*>(out)[e] = o;
}

}  // namespace glue
}  // namespace bi
