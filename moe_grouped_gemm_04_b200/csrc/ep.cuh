// Expert-parallel dispatch into the masked layout, and the combine after it.
//
// The masked layout exists so that the grouped GEMM can meet the
// communication library that moves tokens between the GPUs of an
// expert-parallel group ("DeepGEMM" overview, section "约300行JIT核心", the
// paragraph on MoE layouts); the tokens then travel over NVLink to the GPUs
// that hold their experts and the results travel back (same page, section
// "swapAB与Mega MoE"). These kernels do the data movement on each GPU around
// the exchange, which NCCL's all-to-all performs:
//
//   source GPU: every (token t, choice j) with expert e = topk[t][j] is a
//     "pair"; pairs are ordered by expert, stably by t * k + j (ep_layout),
//     and the quantized token rows with their per-128 scales are copied into
//     that order (ep_pack). The experts of GPU d are [d * G, (d + 1) * G), so
//     the pairs for GPU d are one contiguous segment.
//   exchange: segment d goes to GPU d (rows and scales).
//   destination GPU: the received rows come source by source, each source's
//     rows expert by expert; row i of source s for local expert g goes to slot
//     (rows of g from sources before s) + i of expert g's slab in the masked
//     layout, and masked_m[g] counts them (ep_unpack_masked).
//   after the masked grouped GEMM: the output rows are gathered back into the
//     receive order (ep_gather_rows), exchanged back, and on the source GPU
//     out[t] = bf16(sum_j w[t][j] * y[pair (t, j)]) in fp32, j ascending
//     (ep_combine).
// With a fixed capacity of C rows per destination, segment d starts at row
// d * C of the send buffer and source s's rows at row s * C of the receive
// buffer (equal exchange sizes, known on the host); pairs past C in their
// destination's segment are dropped, and the counts record the pairs sent.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace fg {

constexpr int kEpBlock = 256;
constexpr int kEpMaxTable = 4096;  // source GPUs x local experts (unpack prefix tables, 32 KB)

// Block-wide exclusive prefix of v (0 or 1 per thread) over kEpBlock threads;
// *total gets the block's sum. `scratch` holds kEpBlock / 32 ints.
__device__ __forceinline__ int block_excl_scan(int v, int* scratch, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  int warp_base = 0, sum = 0;
#pragma unroll
  for (int w = 0; w < kEpBlock / 32; ++w) {
    const int s = scratch[w];
    if (w < warp) warp_base += s;
    sum += s;
  }
  __syncthreads();
  *total = sum;
  return warp_base + x - v;
}

// counts[e] = pairs of expert e. Block e counts expert e; block 0 also marks
// the pairs that go nowhere (negative expert: a dropped choice; expert >= E:
// an error, reported as FG_DEVICE_BAD_M_INDEX) with send_pos = -1.
__global__ void __launch_bounds__(kEpBlock) ep_count_kernel(const int32_t* topk, int P, int E,
                                                            int32_t* counts, int32_t* send_pos,
                                                            int* status) {
  grid_dependency_wait();
  __shared__ int red[kEpBlock / 32];
  const int e = blockIdx.x;
  int c = 0;
  bool bad = false;
  for (int p = threadIdx.x; p < P; p += kEpBlock) {
    const int v = topk[p];
    c += v == e ? 1 : 0;
    if (e == 0 && (v < 0 || v >= E)) {
      send_pos[p] = -1;
      bad |= v >= E;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = c;
  if (bad) raise_status(status, 3 /* FG_DEVICE_BAD_M_INDEX */);
  __syncthreads();
  if (threadIdx.x == 0) {
    int s = 0;
    for (int w = 0; w < kEpBlock / 32; ++w) s += red[w];
    counts[e] = s;
  }
}

// send_pos of expert e's pairs: (pairs of experts before e) + the pair's rank
// among expert e's pairs in (t, j) order. Block e handles expert e.
// Fixed capacity (C > 0, G experts per destination GPU): the send buffer
// holds C rows per destination, so the position is (e / G) * C + (pairs of
// the destination's experts before e) + the rank; a pair that would land at
// C or beyond in its destination's segment is dropped (send_pos = -1,
// FG_DEVICE_EP_OVERFLOW).
__global__ void __launch_bounds__(kEpBlock) ep_position_kernel(const int32_t* topk, int P,
                                                               const int32_t* counts, int G, int C,
                                                               int32_t* send_pos, int* status) {
  grid_dependency_wait();
  __shared__ int scratch[kEpBlock / 32];
  __shared__ int base_s;
  const int e = blockIdx.x;
  const int first = C > 0 ? e / G * G : 0;  // first expert of e's segment
  if (threadIdx.x == 0) {
    int b = 0;
    for (int x = first; x < e; ++x) b += counts[x];
    base_s = b;
  }
  __syncthreads();
  int run = base_s;
  bool over = false;
  for (int p0 = 0; p0 < P; p0 += kEpBlock) {
    const int p = p0 + threadIdx.x;
    const int mine = p < P && topk[p] == e ? 1 : 0;
    int total;
    const int ex = block_excl_scan(mine, scratch, &total);
    if (mine) {
      const int i = run + ex;  // position within the segment (C > 0) or the buffer
      if (C > 0 && i >= C) {
        send_pos[p] = -1;
        over = true;
      } else {
        send_pos[p] = C > 0 ? (e / G) * C + i : i;
      }
    }
    run += total;
  }
  if (over) raise_status(status, 6 /* FG_DEVICE_EP_OVERFLOW */);
}

// Fixed capacity: counts[e] becomes the pairs of expert e that are sent,
// i.e. those below C in their destination's rows (the receivers size their
// segments by these counts). One thread per destination, after the position
// kernel has read the full counts.
__global__ void __launch_bounds__(kEpBlock) ep_cap_counts_kernel(int32_t* counts, int E, int G, int C) {
  grid_dependency_wait();
  for (int d = threadIdx.x; d < E / G; d += kEpBlock) {
    int run = 0;
    for (int e = d * G; e < (d + 1) * G; ++e) {
      const int c = counts[e];
      const int room = C - run;
      counts[e] = room <= 0 ? 0 : (c < room ? c : room);
      run += c;
    }
  }
}

// send rows: pair p = t * k + j with send_pos[p] >= 0 copies token row t
// (K bytes) and its K / 128 scales (from the MN-major per-token layout,
// row stride sfa_stride) into row send_pos[p] of the send buffers. One warp
// per pair.
__global__ void __launch_bounds__(kEpBlock) ep_pack_kernel(const uint8_t* q, const float* sfa,
                                                           int sfa_stride, const int32_t* send_pos,
                                                           int P, int k, int K, uint8_t* send_q,
                                                           float* send_s) {
  grid_dependency_wait();
  const int lane = threadIdx.x & 31;
  const int p = blockIdx.x * (kEpBlock / 32) + (threadIdx.x >> 5);
  if (p >= P) return;
  const int pos = send_pos[p];
  if (pos < 0) return;
  const int t = p / k;
  const uint4* src = reinterpret_cast<const uint4*>(q + static_cast<int64_t>(t) * K);
  uint4* dst = reinterpret_cast<uint4*>(send_q + static_cast<int64_t>(pos) * K);
  for (int c = lane; c < K / 16; c += 32) dst[c] = src[c];
  const int KB = K / 128;
  for (int kb = lane; kb < KB; kb += 32)
    send_s[static_cast<int64_t>(pos) * KB + kb] = sfa[static_cast<int64_t>(kb) * sfa_stride + t];
}

// Receive order -> masked layout. recv_counts[s * G + g] = rows source s sent
// for local expert g; the received rows come source by source, expert by
// expert: packed one after another (C = 0, R rows in all), or source s's rows
// from row s * C of a buffer of C rows per source (C > 0, R = W * C, the rows
// after a source's last one unused: recv_slot = -1). Row r of (s, g) at index
// i lands in slot (rows of g from sources before s) + i of expert g; slots
// past M_max are dropped (recv_slot = -1, FG_DEVICE_EP_OVERFLOW). Every block
// builds the prefix tables in shared memory; one warp per received row; block
// 0 writes masked_m.
__global__ void __launch_bounds__(kEpBlock) ep_unpack_kernel(
    const uint8_t* recv_q, const float* recv_s, const int32_t* recv_counts, int W, int G, int C, int R,
    int M_max, int K, uint8_t* A, float* sfa, int32_t* masked_m, int32_t* recv_slot, int* status) {
  grid_dependency_wait();
  __shared__ int off[kEpMaxTable + 1];  // receive-order start of (s, g), flattened s * G + g
  __shared__ int eoff[kEpMaxTable];     // slot of (s, g)'s first row in expert g's slab
  const int SG = W * G;
  if (threadIdx.x == 0) {
    int run = 0;
    bool over = false;
    for (int x = 0; x < SG; ++x) {
      if (C > 0 && x % G == 0) run = (x / G) * C;  // each source's segment starts on its own
      off[x] = run;
      run += recv_counts[x];
      // (a segment never holds more than C rows; counts that say otherwise
      // are reported, and the rows past the segment are never read)
      if (C > 0 && x % G == G - 1 && run > (x / G + 1) * C) over = true;
    }
    off[SG] = C > 0 ? W * C : run;
    if (over && blockIdx.x == 0) raise_status(status, 6 /* FG_DEVICE_EP_OVERFLOW */);
  }
  for (int g = threadIdx.x; g < G; g += kEpBlock) {
    int run = 0;
    for (int s = 0; s < W; ++s) {
      eoff[s * G + g] = run;
      run += recv_counts[s * G + g];
    }
    if (blockIdx.x == 0) {
      if (run > M_max) raise_status(status, 6 /* FG_DEVICE_EP_OVERFLOW */);
      masked_m[g] = run < M_max ? run : M_max;
    }
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * (kEpBlock / 32) + (threadIdx.x >> 5);
  if (r >= R) return;
  int lo = 0, hi = SG;  // off[lo] <= r < off[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (off[mid] <= r) lo = mid; else hi = mid;
  }
  const int g = lo % G;
  const int slot = eoff[lo] + (r - off[lo]);
  // (the unused rows after a source's last one in a fixed-capacity buffer)
  if (r - off[lo] >= recv_counts[lo] || slot >= M_max) {
    if (lane == 0) recv_slot[r] = -1;
    return;
  }
  const int64_t row = static_cast<int64_t>(g) * M_max + slot;
  if (lane == 0) recv_slot[r] = static_cast<int32_t>(row);
  const uint4* src = reinterpret_cast<const uint4*>(recv_q + static_cast<int64_t>(r) * K);
  uint4* dst = reinterpret_cast<uint4*>(A + row * K);
  for (int c = lane; c < K / 16; c += 32) dst[c] = src[c];
  const int KB = K / 128;
  const int stride = (M_max + 3) / 4 * 4;
  for (int kb = lane; kb < KB; kb += 32)
    sfa[(static_cast<int64_t>(g) * KB + kb) * stride + slot] = recv_s[static_cast<int64_t>(r) * KB + kb];
}

// out[r] = D row recv_slot[r] (bf16, N columns), zeros for dropped rows.
__global__ void __launch_bounds__(kEpBlock) ep_gather_kernel(const uint16_t* D, const int32_t* recv_slot,
                                                             int R, int N, uint16_t* out) {
  grid_dependency_wait();
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * (kEpBlock / 32) + (threadIdx.x >> 5);
  if (r >= R) return;
  const int row = recv_slot[r];
  uint4* dst = reinterpret_cast<uint4*>(out + static_cast<int64_t>(r) * N);
  if (row < 0) {
    for (int c = lane; c < N / 8; c += 32) dst[c] = make_uint4(0, 0, 0, 0);
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(D + static_cast<int64_t>(row) * N);
  for (int c = lane; c < N / 8; c += 32) dst[c] = src[c];
}

// out[t][n] = bf16_rne(sum over j ascending of w[t][j] * y[send_pos[t k + j]][n]),
// each term an fp32 fused multiply-add; choices with send_pos < 0 add
// nothing. One block per token, 8 columns (16 bytes) per thread step.
__global__ void __launch_bounds__(kEpBlock) ep_combine_kernel(const uint16_t* y, const int32_t* send_pos,
                                                              const float* w, int k, int N,
                                                              uint16_t* out) {
  grid_dependency_wait();
  const int t = blockIdx.x;
  for (int c = threadIdx.x; c < N / 8; c += kEpBlock) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    for (int j = 0; j < k; ++j) {
      const int pos = send_pos[t * k + j];
      if (pos < 0) continue;
      const float wj = w[t * k + j];
      const uint4 v = reinterpret_cast<const uint4*>(y + static_cast<int64_t>(pos) * N)[c];
      const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] = __fmaf_rn(wj, __uint_as_float(u[i] << 16), acc[2 * i]);
        acc[2 * i + 1] = __fmaf_rn(wj, __uint_as_float(u[i] & 0xFFFF0000u), acc[2 * i + 1]);
      }
    }
    reinterpret_cast<uint4*>(out + static_cast<int64_t>(t) * N)[c] =
        make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                   pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
  }
}

}  // namespace fg
