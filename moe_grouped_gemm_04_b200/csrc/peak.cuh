// FP8 tensor-core rate of this GPU, measured with the same instruction the
// GEMMs issue: one CTA per SM issues tcgen05.mma kind::f8f6f4 (M = 128,
// N = 256, K = 32; four per 128-wide K block) back to back from operand tiles
// that stay in shared memory, into one fp32 accumulator in tensor memory.
// No operand is loaded and nothing is promoted, so the launch runs at the
// rate the tensor pipe sustains under the clock and power limits of the
// moment: the ceiling of every tensor-bound kernel in this library.
//
// The operands are small integers, so the result is exact and the caller can
// check that every MMA ran: a[m][k] = peak_a_value(m, k % 16) and
// b[n][k] = peak_b_value(n, k % 16), both in [-2, 2]; after `iters` K blocks
//   out[cta][m][n] = iters * 8 * sum_{j < 16} peak_a_value(m, j) * peak_b_value(n, j)
// (|entry| <= iters * 512, exact in fp32 for iters <= 32768). Because the
// value depends on k only through k % 16, every 16-byte piece of an operand
// row is the same, and the 128-byte swizzle (which permutes those pieces
// within a row) leaves the operands unchanged.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace fg {

constexpr int kPeakN = 256;         // accumulator columns (MMA N)
constexpr int kPeakGroup = 16;      // K blocks per commit; two groups in flight
constexpr int kPeakMaxIters = 32768;
// more than half of an SM's shared memory, so that no two CTAs share an SM
constexpr int kPeakSmem = 120 * 1024;

__host__ __device__ constexpr int peak_a_value(int m, int j) { return (2 * m + 3 * j) % 5 - 2; }
__host__ __device__ constexpr int peak_b_value(int n, int j) { return (3 * n + 2 * j + n / 16) % 5 - 2; }

// e4m3 codes of -2, -1, 0, 1, 2
__device__ __forceinline__ uint8_t peak_code(int v) {
  return v == 0 ? 0x00 : static_cast<uint8_t>((v < 0 ? 0x80 : 0x00) | (v == 1 || v == -1 ? 0x38 : 0x40));
}

__global__ void __launch_bounds__(128, 1) fp8_mma_peak_kernel(int iters, float* out, int* status,
                                                            uint64_t timeout_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem;              // 128 rows x 128 bytes
  uint8_t* sB = smem + 128 * 128;  // 256 rows x 128 bytes
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + 128 * 128 + kPeakN * 128);
  uint64_t* fin = bar + 2;  // completes once, when every MMA has run
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  for (int i = threadIdx.x; i < 128 * 128; i += 128) sA[i] = peak_code(peak_a_value(i >> 7, i & 15));
  for (int i = threadIdx.x; i < kPeakN * 128; i += 128) sB[i] = peak_code(peak_b_value(i >> 7, i & 15));
  fence_proxy_async_shared();  // the tensor core reads what these generic stores wrote
  if (threadIdx.x == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kPeakN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl ctl{abort_flag, status, timeout_ns};
  const int groups = (iters + kPeakGroup - 1) / kPeakGroup;

  // Group g of K blocks commits to bar[g & 1] (its (g >> 1)-th phase); group
  // g is issued once group g - 2 has completed, so two groups are in flight.
  if (warp == 0) {
    constexpr uint32_t idesc = mma_idesc_e4m3(128, kPeakN);
    const uint64_t adesc = smem_desc_sw128(smem_u32(sA));
    const uint64_t bdesc = smem_desc_sw128(smem_u32(sB));
    for (int g = 0; g < groups; ++g) {
      if (g >= 2 && !warp_wait(&bar[g & 1], ((g - 2) >> 1) & 1u, ctl, lane)) break;
      tc_fence_after();
      if (elect_one()) {
        const int n = min(kPeakGroup, iters - g * kPeakGroup);
        for (int i = 0; i < n; ++i) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_f8(tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (g | i | k) != 0 ? 1u : 0u);
        }
        mma_commit(&bar[g & 1]);
      }
      __syncwarp();
    }
    // (a commit covers every earlier MMA of the issuing thread; the same
    // lane is elected each time in the converged warp)
    if (elect_one()) mma_commit(fin);
    __syncwarp();
  }
  // Every warp waits for the final commit (a barrier that completes once, so
  // a wait that starts early cannot mistake an earlier phase for it), then
  // reads its 32 accumulator rows.
  const bool done = warp_wait(fin, 0u, ctl, lane);
  tc_fence_after();
  if (done) {
    const int row = warp * 32 + lane;
    float* dst = out + (static_cast<int64_t>(blockIdx.x) * 128 + row) * kPeakN;
#pragma unroll 1
    for (int c = 0; c < kPeakN; c += 32) {
      float v[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(c), v);
#pragma unroll
      for (int j = 0; j < 32; j += 4)
        *reinterpret_cast<float4*>(dst + c + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    // MMAs of an abandoned wait may still be running: let them land first
    if (!done && lane == 0) {
      const uint64_t t0 = wait_clock();
      while (!mbar_try_wait(fin, 0u) &&
             wait_clock() - t0 < wait_cycles(20000000ull)) {
      }
    }
    __syncwarp();
    tmem_dealloc(tmem, kPeakN);
  }
}

}  // namespace fg
