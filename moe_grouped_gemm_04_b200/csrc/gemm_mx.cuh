// FP8 e4m3 GEMM with power-of-two (UE8M0) scales for sm_100a: the scales are
// applied inside the tensor core by tcgen05.mma kind::mxf8f6f4.block_scale,
// so the whole K range accumulates in tensor memory and no promotion pass is
// needed.
//
// The operation is the one of gemm.cuh,
//   D[m][n] = sum_kb sa[m][kb] * sb[n/128][kb] * sum_{k in kb} a[m][k] * b[n][k],
// restricted to scales that are powers of two (the UE8M0 scale format:
// DeepSeek-V3 review "28.5 倍压缩 + 1/10 成本", "创新之处" item 4, scales
// rounded to powers of two so that applying one is an exponent shift). With
// such scales every product a * b * sa * sb is exact in fp32, so scaling each
// 32-wide K slice inside the MMA gives the same sum as scaling each 128-wide
// K block after it, up to the order of the fp32 additions. The scales stay
// fp32 in global memory (the layouts of gemm.cuh); the kernel takes their
// exponent bytes.
//
// CTA roles (one CTA per SM, persistent over 128-token x BW-weight tiles):
//   warp 0      producer: lane 0 loads the weight tile, lane 1 the token
//               tile of each K block onto the stage's "full" barrier (TMA);
//               lane 2 the fp32 scales of the stage onto its "sa full"
//               barrier: the 128 token scales with one TMA copy, the (at most
//               three) weight-block scales the tile's rows touch with 4-byte
//               cp.async copies.
//   warp 1      MMA issuer: per K block copies the stage's scale groups from
//               shared to tensor memory (tcgen05.cp) and issues 4 block-scaled
//               MMAs (K = 32 each) into the tile's accumulator; commits the
//               stage to "empty" and, after the last K block, the accumulator
//               to "tmem full".
//   warp 2      scale converter: per K block takes the staged fp32 scales of
//               the tile's 128 token rows and BW weight rows, keeps their
//               exponent bytes (UE8M0 has the fp32 exponent's bias) and writes
//               them in the shared layout tcgen05.cp expects, then arrives on
//               the stage's "sf full" barrier. (Everything it reads is already
//               in shared memory, staged as deep as the operand tiles.)
//   warp 3      idle (keeps the epilogue warps aligned to TMEM lane quadrants)
//   warps 4..   epilogue: per tile, 32 accumulator columns at a time from
//               tensor memory to registers, bf16, a 64-byte-swizzled shared
//               image of 32 rows x 32 columns and a tensor store; the
//               accumulator is released as soon as its last columns are read.
// With two accumulators (BW <= 224) the epilogue of one tile overlaps the
// MMAs of the next; with BW = 256 the MMAs wait for the accumulator to be
// read (8 epilogue warps keep that short).
#pragma once

#include <cstdint>
#include <cuda.h>

#include "gemm.cuh"
#include "ptx.cuh"

namespace fg {

template <int BW_, int STAGES_, int ACC_, int EPQ_>
struct MxCfg {
  static constexpr int BT = 128;          // token rows per tile (MMA M)
  static constexpr int BW = BW_;          // weight rows per tile (MMA N)
  static constexpr bool SWAP = false;     // tile helpers of gemm.cuh: tokens on the lanes
  static constexpr bool PAIR = false;
  static constexpr int STAGES = STAGES_;
  static constexpr int ACC = ACC_;        // accumulators in tensor memory
  static constexpr int EPQ = EPQ_;        // epilogue warps per TMEM lane quadrant
  static_assert(BW % 32 == 0 && BW >= 32 && BW <= 256, "tcgen05 N for M = 128, 32-column chunks");
  static constexpr int EW = 4 * EPQ;      // epilogue warps
  static constexpr int ECOLS = BW / EPQ;  // accumulator columns per epilogue warp
  static_assert(ECOLS % 32 == 0, "epilogue chunks of 32 columns");
  static constexpr int EPI_BASE = 4;      // first epilogue warp
  static constexpr int NUM_THREADS = (EPI_BASE + EW) * 32;
  // scale-factor groups per stage: 128 token rows, ceil(BW / 128) x 128 weight rows
  static constexpr int SFB_GROUPS = (BW + 127) / 128;
  static constexpr int SF_COLS = 4 * (1 + SFB_GROUPS);    // tensor-memory columns per stage
  static constexpr int SF_BYTES = 512 * (1 + SFB_GROUPS);  // shared bytes per stage
  // staged fp32 scales per stage: 128 token scales, then the scales of the
  // (at most NBT) 128-row weight blocks the tile's rows touch
  static constexpr int NBT = SFB_GROUPS + 1;
  static constexpr int RAW_BYTES = 512 + 128;
  static constexpr int TMEM_USED = ACC * BW + STAGES * SF_COLS;
  static_assert(TMEM_USED <= 512, "TMEM has 512 columns");
  static constexpr int TMEM_COLS = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64
                                   : TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
  static constexpr int A_BYTES = BT * 128;
  static constexpr int B_BYTES = BW * 128;
  static constexpr int EPI_RING = 2;         // image buffers per epilogue warp
  static constexpr int BOX_BYTES = 32 * 64;  // 32 rows x 32 bf16 columns
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_SF = OFF_B + STAGES * B_BYTES;
  static constexpr int OFF_RAW = OFF_SF + STAGES * SF_BYTES;  // 128-byte aligned
  static constexpr int OFF_EPI = (OFF_RAW + STAGES * RAW_BYTES + 1023) / 1024 * 1024;
  static constexpr int OFF_BAR = OFF_EPI + EW * EPI_RING * BOX_BYTES;
  static constexpr int NUM_BARS = 4 * STAGES + 2 * ACC;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_TABLE = (OFF_MISC + 16 + 15) / 16 * 16;
  static constexpr int table_bytes(int form) { return form == kFormDense ? 0 : kTableMax * 4; }
  static constexpr int smem_bytes(int form) { return OFF_TABLE + table_bytes(form) + 1024; }

  static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "swizzle atoms");
  static_assert(OFF_SF % 128 == 0 && OFF_RAW % 128 == 0 && RAW_BYTES % 128 == 0,
                "scale groups and staged scales: 128-byte aligned");
  static_assert(NBT * 4 <= RAW_BYTES - 512, "staged weight-block scales");
  static_assert(smem_bytes(kFormContig) <= 232448, "shared memory per CTA");
};

// 16-byte chunk c (columns 8c .. 8c + 7) of row r of a 32-row x 64-byte box
// in the 64-byte swizzled layout of the tensor map: chunk bits 4-5 of the
// offset are XORed with bits 7-8, i.e. with (r / 2) % 4.
__device__ __forceinline__ int sw64_offset(int r, int c) { return r * 64 + ((c ^ ((r >> 1) & 3)) << 4); }

// UE8M0 byte of an fp32 power of two: its biased exponent, replicated into
// the four bytes of a scale word (the MMA reads byte 0).
__device__ __forceinline__ uint32_t ue8m0_word(float s) {
  return ((__float_as_uint(s) >> 23) & 0xFFu) * 0x01010101u;
}

// Bounded wait of a whole warp: lane 0 polls, every lane returns its verdict.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtl& ctl, int lane) {
  int ok = 1;
  if (lane == 0) ok = mbar_wait(bar, parity, ctl) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

template <class C, int FORM>
__global__ void __launch_bounds__(C::NUM_THREADS, 1)
    fp8_gemm_mx_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmD,
                       const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem + C::OFF_A;
  uint8_t* sB = smem + C::OFF_B;
  uint8_t* sSF = smem + C::OFF_SF;
  uint8_t* sRAW = smem + C::OFF_RAW;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + C::STAGES;
  uint64_t* sf_full = empty + C::STAGES;  // the stage's scale groups are written
  uint64_t* sa_full = sf_full + C::STAGES;  // the stage's fp32 scales have landed
  uint64_t* tfull = sa_full + C::STAGES;  // an accumulator holds a finished tile
  uint64_t* tempty = tfull + C::ACC;      // ... and has been read by the epilogue
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  int* table = reinterpret_cast<int*>(smem + C::OFF_TABLE);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 2);      // weight- and token-tile lanes' expect_tx
      mbar_init(&empty[s], 1);     // the MMA commit
      mbar_init(&sf_full[s], 1);   // the converter warp
      mbar_init(&sa_full[s], 2);   // scale lane: expect_tx (TMA) + cp.async arrival
    }
    for (int b = 0; b < C::ACC; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], C::EW);  // one arrival per epilogue warp
    }
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmSA);
    tma_prefetch_desc(&tmD);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  // Everything above may overlap the previous kernel; memory comes after this.
  grid_dependency_wait();
  if (warp == 0) build_table<C, FORM>(p, table, lane);
  tc_fence_before();
  __syncwarp();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tmem_sf = tmem_base + static_cast<uint32_t>(C::ACC * C::BW);
  const WaitCtl ctl{abort_flag, p.status, p.timeout_ns};
  const int total = total_tiles<C, FORM>(p, table);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane < 3) {
      uint32_t it = 0;
      for (int t = blockIdx.x; t < total; t += gridDim.x) {
        const Tile w = resolve_tile<C, FORM>(p, table, t, 0);
        if (!w.valid) continue;
        // weight blocks the tile's rows touch (clamped: rows past N are never stored)
        const int nb0 = (w.nt * C::BW) >> 7;
        const float* sfb_e = p.sfb + static_cast<int64_t>(w.e) * p.NB * p.KB;
        for (int kb = 0; kb < p.KB; ++kb, ++it) {
          const int s = it % C::STAGES;
          if (!mbar_wait(&empty[s], ((it / C::STAGES) & 1u) ^ 1u, ctl)) goto producer_done;
          if (lane == 0) {
            mbar_arrive_expect_tx(&full[s], C::B_BYTES);
            tma_load_2d(sB + s * C::B_BYTES, &tmB, &full[s], kb * 128, w.e * p.N + w.nt * C::BW);
          } else if (lane == 1) {
            mbar_arrive_expect_tx(&full[s], C::A_BYTES);
            tma_load_2d(sA + s * C::A_BYTES, &tmA, &full[s], kb * 128,
                        (FORM == kFormMasked ? w.e * p.M : 0) + w.mt * C::BT);
          } else {
            uint8_t* raw = sRAW + s * C::RAW_BYTES;
            mbar_arrive_expect_tx(&sa_full[s], 512);
            // token scales past M read as zero (their rows are never stored)
            tma_load_2d(raw, &tmSA, &sa_full[s], w.mt * C::BT,
                        (FORM == kFormMasked ? w.e * p.KB : 0) + kb);
#pragma unroll
            for (int j = 0; j < C::NBT; ++j)
              cp_async_4(raw + 512 + 4 * j, sfb_e + static_cast<int64_t>(min(nb0 + j, p.NB - 1)) * p.KB + kb);
            cp_async_mbar_arrive(&sa_full[s]);
          }
        }
      }
    producer_done:
      // the last fill of every stage has landed and been consumed before the
      // CTA releases its shared memory
      if (lane == 0) {
        for (uint32_t s = 0; s < C::STAGES && s < it; ++s) {
          const uint32_t last = (it - 1 - s) / C::STAGES * C::STAGES + s;
          drain_wait(&full[s], (last / C::STAGES) & 1u, kDrainLimitNs);
          drain_wait(&empty[s], (last / C::STAGES) & 1u, kDrainLimitNs);
        }
      } else if (lane == 2) {
        for (uint32_t s = 0; s < C::STAGES && s < it; ++s) {
          const uint32_t last = (it - 1 - s) / C::STAGES * C::STAGES + s;
          drain_wait(&sa_full[s], (last / C::STAGES) & 1u, kDrainLimitNs);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = mma_idesc_e4m3_bs(C::BT, C::BW);
      uint32_t it = 0, tc = 0;
      for (int t = blockIdx.x; t < total; t += gridDim.x) {
        const Tile w = resolve_tile<C, FORM>(p, table, t, 0);
        if (!w.valid) continue;
        const int b = tc % C::ACC;
        if (!mbar_wait(&tempty[b], ((tc / C::ACC) & 1u) ^ 1u, ctl)) goto mma_done;
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(b * C::BW);
        for (int kb = 0; kb < p.KB; ++kb, ++it) {
          const int s = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1u;
          if (!mbar_wait(&full[s], ph, ctl)) goto mma_done;
          if (!mbar_wait(&sf_full[s], ph, ctl)) goto mma_done;
          tc_fence_after();
          // the stage's scale groups into its own tensor-memory columns
          // (a copy is ordered before the MMAs this thread issues after it)
          const uint32_t sf = tmem_sf + static_cast<uint32_t>(s * C::SF_COLS);
          const uint32_t sf_smem = smem_u32(sSF + s * C::SF_BYTES);
          tmem_cp_sf_group(sf, sf_smem);
#pragma unroll
          for (int g = 0; g < C::SFB_GROUPS; ++g)
            tmem_cp_sf_group(sf + 4 + 4 * g, sf_smem + 512 * (1 + g));
          const uint64_t adesc = smem_desc_sw128(smem_u32(sA + s * C::A_BYTES));
          const uint64_t bdesc = smem_desc_sw128(smem_u32(sB + s * C::B_BYTES));
#pragma unroll
          for (int k = 0; k < 4; ++k)  // 32 bytes (= 32 e4m3 along K) per MMA
            mma_f8_bs(d, adesc + 2 * k, bdesc + 2 * k, idesc, sf, sf + 4, (kb | k) != 0 ? 1u : 0u);
          mma_commit(&empty[s]);
        }
        mma_commit(&tfull[b]);
        ++tc;
      }
    mma_done:
      if (tc > 0) drain_wait(&tfull[(tc - 1) % C::ACC], ((tc - 1) / C::ACC) & 1u, kDrainLimitNs);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ scale converter
    uint32_t it = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const Tile w = resolve_tile<C, FORM>(p, table, t, 0);
      if (!w.valid) continue;
      // staged weight-block index of this lane's weight rows lane + 32 r1 + 128 g
      const int n0 = w.nt * C::BW;
      int jb[C::SFB_GROUPS][4];
#pragma unroll
      for (int g = 0; g < C::SFB_GROUPS; ++g)
#pragma unroll
        for (int r1 = 0; r1 < 4; ++r1) jb[g][r1] = ((n0 + 128 * g + 32 * r1 + lane) >> 7) - (n0 >> 7);
      for (int kb = 0; kb < p.KB; ++kb, ++it) {
        const int s = it % C::STAGES;
        // the stage's scales have landed (and, since the producer refilled the
        // stage, its previous scale groups have been copied out)
        if (!warp_wait(&sa_full[s], (it / C::STAGES) & 1u, ctl, lane)) goto convert_done;
        const float* raw = reinterpret_cast<const float*>(sRAW + s * C::RAW_BYTES);
        uint8_t* grp = sSF + s * C::SF_BYTES + lane * 16;
        *reinterpret_cast<uint4*>(grp) = make_uint4(ue8m0_word(raw[lane]), ue8m0_word(raw[lane + 32]),
                                                    ue8m0_word(raw[lane + 64]), ue8m0_word(raw[lane + 96]));
#pragma unroll
        for (int g = 0; g < C::SFB_GROUPS; ++g)
          *reinterpret_cast<uint4*>(grp + 512 * (1 + g)) =
              make_uint4(ue8m0_word(raw[128 + jb[g][0]]), ue8m0_word(raw[128 + jb[g][1]]),
                         ue8m0_word(raw[128 + jb[g][2]]), ue8m0_word(raw[128 + jb[g][3]]));
        fence_proxy_async_shared();  // visible to tcgen05.cp (async proxy)
        __syncwarp();
        if (lane == 0) mbar_arrive(&sf_full[s]);
      }
    }
  convert_done:;
  } else if (warp >= C::EPI_BASE) {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - C::EPI_BASE;
    const int quad = warp & 3;          // TMEM lanes this warp may access
    const int c0 = (ew >> 2) * C::ECOLS;
    const int row = quad * 32 + lane;   // token row of the tile
    const uint32_t t_lane = static_cast<uint32_t>(quad * 32) << 16;
    uint8_t* ring = smem + C::OFF_EPI + ew * C::EPI_RING * C::BOX_BYTES;
    uint32_t tc = 0, boxes = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const Tile w = resolve_tile<C, FORM>(p, table, t, 0);
      if (!w.valid) continue;
      int m_valid = p.M;
      if (FORM == kFormMasked) {
        m_valid = __ldg(p.masked_m + w.e);
        m_valid = m_valid < 0 ? 0 : (m_valid > p.M ? p.M : m_valid);
      }
      const int m = w.mt * C::BT + row;
      int row_mi = 0;
      if (FORM == kFormContig) row_mi = m < p.M ? __ldg(p.m_indices + m) : -1;
      const bool ok = m < m_valid && (FORM != kFormContig || row_mi >= 0);
      // a warp whose 32 rows are all stored writes through tensor stores
      const bool staged = __all_sync(0xffffffffu, ok);
      const int y = (FORM == kFormMasked ? w.e * p.M : 0) + w.mt * C::BT + quad * 32;
      const int b = tc % C::ACC;
      if (!warp_wait(&tfull[b], (tc / C::ACC) & 1u, ctl, lane)) goto epi_done;
      tc_fence_after();
#pragma unroll 1
      for (int ch = 0; ch < C::ECOLS / 32; ++ch) {
        uint32_t r[32];
        tmem_ld32_issue(tmem_base + t_lane + static_cast<uint32_t>(b * C::BW + c0 + ch * 32), r);
        tmem_wait_ld32(r);
        if (ch == C::ECOLS / 32 - 1) {
          // the accumulator is in registers: the next tile's MMAs may start
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[b]);
        }
        if (staged) {
          uint8_t* img = ring + (boxes % C::EPI_RING) * C::BOX_BYTES;
          // the tensor store that last used this buffer has read it
          if (boxes >= C::EPI_RING && lane == 0) bulk_wait_group_read<C::EPI_RING - 1>();
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4*>(img + sw64_offset(lane, c)) = make_uint4(
                pack_bf16x2(__uint_as_float(r[8 * c + 0]), __uint_as_float(r[8 * c + 1])),
                pack_bf16x2(__uint_as_float(r[8 * c + 2]), __uint_as_float(r[8 * c + 3])),
                pack_bf16x2(__uint_as_float(r[8 * c + 4]), __uint_as_float(r[8 * c + 5])),
                pack_bf16x2(__uint_as_float(r[8 * c + 6]), __uint_as_float(r[8 * c + 7])));
          fence_proxy_async_shared();
          __syncwarp();
          if (lane == 0) {
            const int x = w.nt * C::BW + c0 + ch * 32;
            if (x < p.N) tma_store_2d(&tmD, img, x, y);  // columns past N are clipped
            bulk_commit_group();  // (possibly empty: keeps one group per buffer use)
          }
          ++boxes;
        } else {
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
          store_tile_part<C, FORM, 32>(p, w, row, c0 + ch * 32, v, m_valid, row_mi);
        }
      }
      ++tc;
    }
  epi_done:
    // this warp's tensor stores have finished reading shared memory
    if (lane == 0) bulk_wait_group_read<0>();
  }

  // ---------------------------------------------------------------- teardown
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  grid_launch_dependents();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace fg
