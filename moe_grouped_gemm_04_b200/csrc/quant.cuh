// FP8 quantizers: per-token (1x128) activation scaling and per-block (128x128)
// weight scaling. Both are HBM-bound streams: 2 bytes read and 1 byte written
// per element plus one fp32 scale per group. Loads are 16-byte vectors,
// code stores 16-byte (per token) or 8-byte (per block) vectors; the amax reduction is a warp shuffle (per token) or a
// warp shuffle plus a shared-memory step (per block).
//
// Arithmetic (must match the oracle bit for bit):
//   amax_c = max(amax, 1e-4f); scale = amax_c / 448 (IEEE division);
//   code = cvt.rn.satfinite.e4m3(x * (448 / amax_c)) with one fp32 multiply;
// or, with power-of-two (UE8M0) scales, scale = the smallest power of two at
// or above amax_c / 448 and code = cvt.rn.satfinite.e4m3(x / scale), exact.
// Sources: "DeepGEMM" overview (zixun.chuxinyishu.com/article/345.html),
// section "FP8与细粒度缩放" (per-slice activation and per-block weight
// scales); DeepSeek-V3 review (developer.cloud.tencent.cn/article/2686109),
// "创新之处" item 4 (one scale per 128 elements, 128x128 blocks) and
// "风险与不足" item 6 (the 448.0 bound).
#pragma once

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <cstdint>

#include "ptx.cuh"

namespace fg {

constexpr float kFp8Max = 448.0f;
constexpr float kAmaxFloor = 1e-4f;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// 8 bf16 values (one 16-byte word) -> 8 e4m3 codes (one 8-byte word).
__device__ __forceinline__ uint2 quantize8(uint4 w, float inv) {
  const uint32_t in[4] = {w.x, w.y, w.z, w.w};
  uint32_t out[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint16_t p0 = cvt_e4m3x2(__fmul_rn(bf16_lo(in[2 * i]), inv),
                                   __fmul_rn(bf16_hi(in[2 * i]), inv));
    const uint16_t p1 = cvt_e4m3x2(__fmul_rn(bf16_lo(in[2 * i + 1]), inv),
                                   __fmul_rn(bf16_hi(in[2 * i + 1]), inv));
    out[i] = static_cast<uint32_t>(p0) | (static_cast<uint32_t>(p1) << 16);
  }
  return make_uint2(out[0], out[1]);
}

// Scale and its reciprocal for a group with amax_c = max(amax, 1e-4).
// UE8M0 = false: s = amax_c / 448, inv = 448 / amax_c (IEEE divisions).
// UE8M0 = true: s = the smallest power of two at or above amax_c / 448 (from
// the fp32 bits of the quotient: 2^E if its mantissa field is zero, else
// 2^(E+1)), inv = 1 / s exactly (biased exponent 254 - e), so that x * inv
// equals x / s. A slice holding an infinity has s = +inf and inv = 0, which
// is x / s as well: finite elements give (signed) zero codes, infinities NaN.
// (For finite bf16 input E stays far below 254: amax / 448 < 2^120.)
template <bool UE8M0>
__device__ __forceinline__ void group_scale(float amx, float& scale, float& inv) {
  if constexpr (UE8M0) {
    const uint32_t u = __float_as_uint(__fdiv_rn(amx, kFp8Max));
    const uint32_t e = ((u >> 23) & 0xFFu) + ((u & 0x007FFFFFu) != 0 ? 1u : 0u);
    scale = __uint_as_float((e > 255u ? 255u : e) << 23);
    inv = e >= 255u ? 0.0f : __uint_as_float((254u - e) << 23);
  } else {
    scale = __fdiv_rn(amx, kFp8Max);
    inv = __fdiv_rn(kFp8Max, amx);
  }
}

__device__ __forceinline__ float amax8(uint4 w) {
  const uint32_t in[4] = {w.x, w.y, w.z, w.w};
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m = fmaxf(m, fabsf(bf16_lo(in[i])));
    m = fmaxf(m, fabsf(bf16_hi(in[i])));
  }
  return m;
}

// One 128-element slice per 8 consecutive threads (16 elements, two 16-byte
// loads each), so that a warp covers 4 adjacent slices of one token row per
// step. A work item is QROW_STEPS such steps of one row (8 slices, 2 KB of
// bf16); warps take items grid-stride, so the only index arithmetic is one
// division per item, and all of an item's loads are issued before any is
// used (4 x 16 bytes in flight per thread). Small inputs still spread over
// many warps (a 64-token row set is 64 x 7 items for K = 7168). The codes of
// a slice leave as one 16-byte store per thread; its scale as one 4-byte
// store into the MN-major layout.
constexpr int QROW_STEPS = 2;  // warp steps (4 slices each) per work item
constexpr int QROW_ITEM = 4 * QROW_STEPS;  // slices per work item

template <bool UE8M0>
__global__ void __launch_bounds__(256) per_token_cast_kernel(const uint16_t* __restrict__ x,
                                                             uint8_t* __restrict__ q,
                                                             float* __restrict__ sfa, int G,
                                                             int M, int K, int stride) {
  // the next kernel may start its prologue now; it waits for this grid
  // before touching memory
  grid_launch_dependents();
  grid_dependency_wait();
  const int KB = K / 128;
  const int chunks = (KB + QROW_ITEM - 1) / QROW_ITEM;
  const int64_t items = static_cast<int64_t>(G) * M * chunks;
  const int lane = threadIdx.x & 31;
  const int grp = lane >> 3;  // slice of the warp step
  const int sub = lane & 7;   // 16 elements of the slice
  const int64_t first = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t step = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  // the loop bound is uniform across a warp (the shuffles below need every lane)
  for (int64_t it = first; it < items; it += step) {
    const int64_t r = it / chunks;  // g * M + m
    const int kb0 = static_cast<int>(it % chunks) * QROW_ITEM;
    const int g = static_cast<int>(r / M), m = static_cast<int>(r % M);
    const uint16_t* xr = x + r * K;
    uint8_t* qr = q + r * K;
    uint4 lo[QROW_STEPS], hi[QROW_STEPS];
#pragma unroll
    for (int u = 0; u < QROW_STEPS; ++u) {
      const int kb = kb0 + u * 4 + grp;
      if (kb < KB) {
        const uint4* src = reinterpret_cast<const uint4*>(xr + kb * 128 + sub * 16);
        lo[u] = __ldg(src);
        hi[u] = __ldg(src + 1);
      } else {
        lo[u] = make_uint4(0, 0, 0, 0);
        hi[u] = lo[u];
      }
    }
#pragma unroll
    for (int u = 0; u < QROW_STEPS; ++u) {
      const int kb = kb0 + u * 4 + grp;
      float a = fmaxf(amax8(lo[u]), amax8(hi[u]));
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 4));
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
      if (kb < KB) {
        float scale, inv;
        group_scale<UE8M0>(fmaxf(a, kAmaxFloor), scale, inv);
        const uint2 c0 = quantize8(lo[u], inv), c1 = quantize8(hi[u], inv);
        *reinterpret_cast<uint4*>(qr + kb * 128 + sub * 16) = make_uint4(c0.x, c0.y, c1.x, c1.y);
        if (sub == 0) sfa[(static_cast<int64_t>(g) * KB + kb) * stride + m] = scale;
      }
    }
  }
}

// One CTA (256 threads) per 128x128 block. Thread t covers rows t/16 + 16*i
// (i = 0..7) and the 8 columns starting at (t%16)*8 of the block.
template <bool UE8M0>
__global__ void __launch_bounds__(256) per_block_cast_kernel(const uint16_t* __restrict__ x,
                                                             uint8_t* __restrict__ q,
                                                             float* __restrict__ sfb, int G,
                                                             int N, int K) {
  __shared__ float warp_max[8];
  grid_dependency_wait();
  grid_launch_dependents();
  const int KB = K / 128;
  const int NB = (N + 127) / 128;
  const int64_t blk = blockIdx.x;
  const int kb = static_cast<int>(blk % KB);
  const int nb = static_cast<int>((blk / KB) % NB);
  const int64_t g = blk / (static_cast<int64_t>(KB) * NB);
  const int col = (threadIdx.x & 15) * 8;
  const int r0 = threadIdx.x >> 4;
  uint4 w[8];
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int n = nb * 128 + r0 + 16 * i;
    if (n < N) {
      const int64_t off = (g * N + n) * K + static_cast<int64_t>(kb) * 128 + col;
      w[i] = __ldg(reinterpret_cast<const uint4*>(x + off));
      a = fmaxf(a, amax8(w[i]));
    } else {
      w[i] = make_uint4(0, 0, 0, 0);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = a;
  __syncthreads();
  a = warp_max[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) a = fmaxf(a, warp_max[i]);
  float scale, inv;
  group_scale<UE8M0>(fmaxf(a, kAmaxFloor), scale, inv);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int n = nb * 128 + r0 + 16 * i;
    if (n < N) {
      const int64_t off = (g * N + n) * K + static_cast<int64_t>(kb) * 128 + col;
      *reinterpret_cast<uint2*>(q + off) = quantize8(w[i], inv);
    }
  }
  if (threadIdx.x == 0) sfb[blk] = scale;
}

// Weight dequantization, the third kernel of the FP8 trio (quantize,
// dequantize, GEMM) the DeepSeek-V3 review describes ("创新之处" item 4):
//   x = bf16(fp32(e4m3(q) * s)), s the fp32 scale of q's 128x128 block,
// both roundings to nearest even (e4m3 -> half -> float is exact). HBM-bound:
// 1 byte read and 2 written per element. A thread converts 16 consecutive
// codes of one row (K % 128 == 0 keeps them inside one block): one 16-byte
// load, two 16-byte stores (one chunk per thread and pass measured faster
// than several loads in flight with fewer threads).
__global__ void __launch_bounds__(256) per_block_dequant_kernel(const uint8_t* __restrict__ q,
                                                                const float* __restrict__ sfb,
                                                                uint16_t* __restrict__ x, int G,
                                                                int N, int K) {
  grid_launch_dependents();
  grid_dependency_wait();
  const int KB = K / 128;
  const int NB = (N + 127) / 128;
  const int64_t chunks = static_cast<int64_t>(G) * N * (K / 16);
  for (int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c < chunks;
       c += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t off = c * 16;
    const int64_t row = off / K;  // g * N + n
    const int k = static_cast<int>(off - row * K);
    const int64_t g = row / N;
    const int n = static_cast<int>(row - g * N);
    const float sc = __ldg(sfb + (g * NB + n / 128) * KB + k / 128);
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(q + off));
    const uint32_t in[4] = {w.x, w.y, w.z, w.w};
    uint32_t out[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      // codes 2i (low byte) and 2i + 1
      const __nv_fp8x2_storage_t pair =
          static_cast<__nv_fp8x2_storage_t>((in[i / 2] >> (16 * (i % 2))) & 0xFFFFu);
      const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
      const float lo = __half2float(__ushort_as_half(h.x));
      const float hi = __half2float(__ushort_as_half(h.y));
      out[i] = pack_bf16x2(__fmul_rn(lo, sc), __fmul_rn(hi, sc));
    }
    uint4* dst = reinterpret_cast<uint4*>(x + off);
    dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
    dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
  }
}

}  // namespace fg
