// Chain probe: cycles per tcgen05.mma.kind::f16 (128 x N x 16, bf16 operands in
// shared memory, fp32 accumulator in tensor memory) when every MMA accumulates into
// the tile the previous one wrote (one chain), and when 2, 4 or 8 independent
// accumulators are interleaved, for N = 32, 64, 128, 192, 224, 256. One CTA on one SM; the
// operands are zeros (their values do not change the timing); clock64() around the
// issue loop and around the completion (tcgen05.commit -> mbarrier).
//
// Every output element of bi_matmul is one such chain of K/16 dependent MMAs (that
// single chain is what makes its bits independent of the batch), so the per-MMA
// latency of one chain bounds the time of any output tile from below.
//
// Build and run on a B200 (prints one JSON line per configuration):
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -std=c++17 \
//        -o mma_chain invariant_deterministic_04_b200/probes/mma_chain.cu && ./mma_chain
#include "../csrc/device.cuh"
#include <cstdio>
using namespace bi;
__device__ __forceinline__ uint64_t sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// smem: A 16 KiB (128 rows x 128 B), B 32 KiB (256 rows x 128 B), barrier.
// unrolled = 0: one MMA per loop trip, descriptors advanced in the loop;
// unrolled = 1: as the matmul kernel issues them, four MMAs (k = 0, 16, 32, 48 of a
// 64-wide block) with precomputed descriptors per trip;
// unrolled = 2: the matmul's whole per-block sequence with the data already present:
// a wait on a stage barrier that is already complete, the fence, the four MMAs, and
// a tcgen05.commit of the stage to a barrier nobody waits on;
// unrolled = 3: the same without the commit; 4: without the wait and the fence;
// 5: the fence and the four MMAs only.
__global__ void __launch_bounds__(128, 1) lat_kernel(int m_instr, int n_instr, int chains, int iters, int unrolled,
                                                      long long* out) {
  extern __shared__ __align__(1024) uint8_t sm[];
  const uint32_t base = (smem_u32(sm) + 1023u) & ~1023u;
  uint8_t* g = sm + (base - smem_u32(sm));
  __shared__ uint32_t tslot;
  __shared__ __align__(8) uint64_t bar, bar_full, bar_empty;
  for (int i = threadIdx.x; i < (16384 + 32768) / 16; i += 128) reinterpret_cast<uint4*>(g)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    mbar_init(smem_u32(&bar_full), 1);   // never arrived on: its previous phase counts as complete
    mbar_init(smem_u32(&bar_empty), 1);
    fence_mbar_init();
  }
  fence_proxy_async_smem();
  if (threadIdx.x < 32) { tmem_alloc(smem_u32(&tslot), 512); tmem_relinquish(); }
  tc_fence_before(); __syncthreads(); tc_fence_after();
  const uint32_t tmem = tslot;
  if (threadIdx.x == 0) {
    const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n_instr >> 3) << 17) |
                           ((uint32_t)(m_instr >> 4) << 24);
    const uint64_t ad = sw128(base), bd = sw128(base + 16384);
    for (int c = 0; c < chains; ++c) tc_mma_f16(tmem + c * n_instr, ad, bd, idesc, 0u);
    tc_commit(smem_u32(&bar));
    mbar_wait(smem_u32(&bar), 0);
    long long t0, t1;
    if (!unrolled) {
      t0 = clock64();
      for (int i = 0; i < iters; ++i)
        for (int c = 0; c < chains; ++c) tc_mma_f16(tmem + c * n_instr, ad + ((i & 3) * 2), bd + ((i & 3) * 2), idesc, 1u);
      t1 = clock64();
    } else if (unrolled >= 2) {
      uint64_t a4[4], b4[4];
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) { a4[kk] = sw128(base + kk * 32); b4[kk] = sw128(base + 16384 + kk * 32); }
      t0 = clock64();
      for (int i = 0; i < iters; i += 4)
        for (int c = 0; c < chains; ++c) {
          if (unrolled == 2 || unrolled == 3) mbar_wait(smem_u32(&bar_full), 1u);
          if (unrolled != 4) tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) tc_mma_f16(tmem + c * n_instr, a4[kk], b4[kk], idesc, 1u);
          if (unrolled == 2 || unrolled == 4) tc_commit(smem_u32(&bar_empty));
        }
      t1 = clock64();
    } else {
      uint64_t a4[4], b4[4];
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) { a4[kk] = sw128(base + kk * 32); b4[kk] = sw128(base + 16384 + kk * 32); }
      t0 = clock64();
      for (int i = 0; i < iters; i += 4)
        for (int c = 0; c < chains; ++c) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) tc_mma_f16(tmem + c * n_instr, a4[kk], b4[kk], idesc, 1u);
        }
      t1 = clock64();
    }
    tc_commit(smem_u32(&bar));
    mbar_wait(smem_u32(&bar), 1);
    const long long t2 = clock64();
    out[0] = t1 - t0;  // issue time
    out[1] = t2 - t0;  // completion time
  }
  tc_fence_before(); __syncthreads();
  if (threadIdx.x < 32) { tc_fence_after(); tmem_dealloc(tmem, 512); }
}
int main() {
  long long* d; cudaMalloc(&d, 16);
  cudaFuncSetAttribute(lat_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 50 * 1024);
  const int iters = 256;
  int ns[] = {32, 64, 128, 192, 224, 256};
  for (int unrolled = 0; unrolled < 6; ++unrolled)
    for (int m : {128, 64})
      for (int n : ns)
        for (int chains = 1; chains <= 8; chains *= 2) {
          if (chains * n > 512) continue;
          if (m == 64 && chains > 1) continue;
          lat_kernel<<<1, 128, 50 * 1024>>>(m, n, chains, iters, unrolled, d);
          long long h[2] = {0, 0};
          cudaError_t e = cudaMemcpy(h, d, 16, cudaMemcpyDeviceToHost);
          if (e != cudaSuccess) { printf("error %s\n", cudaGetErrorString(e)); return 1; }
          printf("{\"M\": %d, \"N\": %d, \"chains\": %d, \"unrolled\": %d, \"iters\": %d, \"issue_cycles\": %lld, "
                 "\"done_cycles\": %lld, \"cycles_per_mma\": %.1f, \"execution_cycles_per_mma\": %.1f}\n",
                 m, n, chains, unrolled, iters, h[0], h[1], (double)h[1] / (iters * chains), m * n / 256.0);
        }
  return 0;
}
