// FP8 e4m3 block-scaled GEMM for sm_100a: tcgen05 MMAs into tensor memory,
// per-128-K promotion into fp32 registers, persistent tile scheduling over the
// dense, contiguous-grouped and masked-grouped layouts.
//
// The operation (two-level accumulation) follows "一文看懂 DeepSeek 開源項目第三彈"
// (animattoys.com), section "為現代 AI 計算而造" and the deployment guide's
// note on promotion, and the "DeepGEMM" overview (zixun.chuxinyishu.com/
// article/345.html), section "FP8与细粒度缩放":
//   D[m][n] = sum_kb sa[m][kb] * sb[n/128][kb] * P_kb[m][n],
//   P_kb[m][n] = sum_{k in block kb} a[m][k] * b[n][k]   (FP8 products, fp32)
// The grouped layouts follow the same page's paragraph on contiguous and
// masked MoE grouping, and the swapped product (D^T = B A^T for thin M) its
// section "swapAB与Mega MoE".
//
// CTA roles (one CTA per SM, persistent over output tiles):
//   producer    TMA: per K block one thread loads the weight tile, one the
//               token tile and one the token scales, each onto the stage's
//               barrier. In the 8-warp form they are lane 0 of warps 0, 2 and
//               3 (three lanes of one warp diverge, and a lane waiting for its
//               stage to be released stalled the other two: the producer then
//               ran barely one stage ahead of the MMA); in the 4-warp form
//               lanes 0..2 of warp 0.
//   warp 1      MMA issuer (converged warp, one elected lane issues): 4 x
//               tcgen05.mma (K = 32 each) per K block into one of two TMEM
//               partial buffers, then commits to the stage's "empty" barrier
//               and the buffer's "tmem full" barrier.
//   promotion warps (2..5, or 4..11 in the 8-warp form, where warpgroup 0
//   holds the producer and MMA roles and gives registers to the promotion
//   warpgroups): per K block read the partial from TMEM
//               (tcgen05.ld), add partial * (sa * sb) into fp32 registers
//               (sb, one value per 128 weight rows and K block, is read from
//               global memory one stage ahead), release the TMEM buffer and
//               the stage; after the last K block round to bf16 and store D.
//               Normal form: a warp whose 32 token rows are all stored writes
//               its slice in one pass into a swizzled shared-memory image and
//               sends it with tensor stores, which drain while the warp
//               promotes the next tile.
// Two TMEM buffers let the MMA of block kb+1 run while block kb is promoted.
//
// Normal form: MMA M = 128 token rows, MMA N = BW weight rows (TMEM lane =
// token, column = weight). Swapped form: MMA M = 128 weight rows, MMA N = BT
// tokens (TMEM lane = weight, column = token), used when M is small.
//
// Split-K (SPLIT > 1): the K blocks of one output tile are dealt round robin
// to the SPLIT CTAs of a thread-block cluster (CTA r takes kb = r, r + SPLIT,
// ...), so that at any moment the cluster reads adjacent 128-byte pieces of
// the same weight rows. The fp32 partial tiles are then reduce-scattered
// through distributed shared memory: CTA j owns token rows
// [j * SLICE_M, (j + 1) * SLICE_M); every CTA pushes its partial values of
// those rows into CTA j's receive slot for that sender with st.async, whose
// bytes count down CTA j's "red_ready" mbarrier (no round trips). CTA j then
// sums its slots in split order and stores its slice of D, so the result
// does not depend on which CTA finishes first.
//
// Programmatic dependent launch: the prologue (barrier init, TMEM
// allocation, descriptor prefetch) may overlap the previous kernel of the
// stream; every global-memory access comes after griddepcontrol.wait.
#pragma once

#include <cstdint>
#include <cuda.h>

#include "ptx.cuh"

namespace fg {

enum : int { kFormDense = 0, kFormContig = 1, kFormMasked = 2, kFormKGrouped = 3 };

constexpr int kTableMax = 2048;  // contiguous: token tiles; masked: experts + 1
constexpr uint64_t kDrainLimitNs = 20000000ull;  // 20 ms for in-flight copies at teardown

struct GemmParams {
  int M;       // rows of one token slab: dense M, contiguous M_total, masked M_max
  int N, K, G;
  int KB;      // K / 128
  int NB;      // ceil(N / 128)
  int num_mt;  // token tiles per slab
  int num_nt;  // weight tiles
  const float* sfb;
  uint16_t* D;
  const int32_t* m_indices;
  const int32_t* masked_m;
  int* status;
  uint64_t timeout_ns;
  // fused expert-FFN epilogue of the block-scaled kernel (otherwise unused):
  // quantized activations h [rows][I] with their per-token scales (MN-major,
  // row stride sfh_stride) and, optionally, the bf16 gate/up values [rows][2I]
  uint8_t* hq;
  float* sfh;
  uint16_t* gu;
  int I;
  int sfh_stride;
  // K-grouped GEMM of the block-scaled kernel: token counts per expert
  // (device) and the fp32 output [G][M][N]
  const int32_t* ks;
  float* d32;
  // one-kernel expert FFN (both GEMMs in one persistent launch): the second
  // GEMM's weight rows (H), K blocks (I / 128), weight-block rows and tiles,
  // its weight-block scales, and the per-token-tile ready counters in global
  // scratch (zero at launch; the first GEMM's epilogue warps count up, the
  // second GEMM's loads of a token tile wait for ready_target)
  int N2, KB2, NB2, num_nt2;
  const float* sfb2;
  int* ready;
  int ready_target;
};

template <int BT_, int BW_, bool SWAP_, int STAGES_, int PW_, int SPLIT_, int KPS_ = 2,
          bool PAIR_ = false>
struct GemmCfg {
  static constexpr int BT = BT_;          // token rows per tile
  static constexpr int BW = BW_;          // weight rows per tile
  static constexpr bool SWAP = SWAP_;
  static constexpr int STAGES = STAGES_;
  static constexpr int PW = PW_;          // promotion warps
  static constexpr int SPLIT = SPLIT_;    // CTAs per cluster sharing one tile's K blocks
  static constexpr int KPS = KPS_;        // K blocks per pipeline stage
  // Pair MMA (tcgen05 cta_group::2): the two CTAs of a cluster compute one
  // tile of 2 * BT tokens x BW weights; each loads its BT token rows and half
  // of the BW weight rows, the leader issues the MMAs, and each CTA's tensor
  // memory receives its own BT x BW slice, which it promotes and stores.
  static constexpr bool PAIR = PAIR_;
  static_assert(!PAIR || (!SWAP && SPLIT == 1 && KPS == 1), "pair MMA: normal form, no split-K");
  static constexpr int CLUSTER = PAIR ? 2 : SPLIT;  // CTAs per cluster
  static constexpr int B_ROWS = PAIR ? BW / 2 : BW;  // weight rows this CTA loads per tile
  static constexpr int MMA_M = PAIR ? 256 : 128;
  static constexpr int MMA_N = SWAP ? BT : BW;
  static_assert(SWAP ? (BW == 128) : (BT == 128), "the lane operand has 128 rows");
  static_assert(MMA_N % 16 == 0 && MMA_N >= 16 && MMA_N <= 256, "tcgen05 N for M = 128");
  static_assert(PW % 4 == 0, "promotion warps cover the 4 TMEM lane quadrants");
  static constexpr int WPQ = PW / 4;      // promotion warps per lane quadrant
  static constexpr int COLS = MMA_N / WPQ;
  static_assert(COLS % 8 == 0, "columns per promotion thread");
  static_assert(SWAP || (COLS <= 128 && (128 % COLS == 0)), "one weight scale per thread");
  static constexpr int A_BYTES = BT * 128;
  static constexpr int B_BYTES = B_ROWS * 128;
  static constexpr int SA_BYTES = BT * 4;                       // one TMA box of token scales
  static constexpr int SA_STAGE = (SA_BYTES + 127) / 128 * 128;  // TMA smem destinations: 128-B aligned
  static constexpr int STAGE_A = KPS * A_BYTES;
  static constexpr int STAGE_B = KPS * B_BYTES;
  static constexpr int STAGE_SA = KPS * SA_STAGE;
  static constexpr int TMEM_USED = 2 * KPS * MMA_N;  // two stages of KPS partial tiles
  static constexpr int TMEM_COLS = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64
                                   : TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
  static_assert(TMEM_USED <= 512, "TMEM has 512 columns");
  static constexpr int PW_BASE = PW == 8 ? 4 : 2;  // first promotion warp
  static constexpr int NUM_THREADS = (PW_BASE + PW) * 32;
  // the whole register file for the one CTA of an SM (allocation in steps of 8)
  static constexpr int MAX_REGS = (65536 / NUM_THREADS) / 8 * 8 > 255 ? 255 : (65536 / NUM_THREADS) / 8 * 8;
  // 8 promotion warps: warpgroup 0 (the producer and MMA warps) drops to
  // REG_LOW registers and the two promotion warpgroups rise to REG_HIGH; the
  // shares add up to the launch allocation of MAX_REGS per thread.
  static constexpr bool REG_SPLIT = PW == 8;
  static constexpr int REG_LOW = 40;
  static constexpr int REG_HIGH = 232;
  static_assert(!REG_SPLIT || 128 * REG_LOW + PW * 32 * REG_HIGH <= NUM_THREADS * MAX_REGS,
                "register split exceeds the launch allocation");
  static constexpr int SAS = 2 * STAGES;  // token-scale ring (read by the promotion warps)
  // split-K receive slots: SPLIT - 1 slots (one per peer; a CTA keeps its own
  // values in registers) of SLICE_M token rows x 128 weights in fp32, stored
  // as groups of 4 consecutive tokens with the weight (TMEM lane) next, so
  // that the 16-byte pushes of a warp land contiguously:
  //   slot[token / 4][weight][token % 4]
  static_assert(SPLIT == 1 || (SWAP && PW == 4 && (SPLIT == 2 || SPLIT == 4 || SPLIT == 8)),
                "split-K: swapped form, 128 promotion threads, 2, 4 or 8 CTAs");
  static constexpr int TN = SWAP ? 128 : BW;  // weight columns of a tile
  static constexpr int SLICE_M = BT / SPLIT;
  static constexpr int SLOT_FLOATS = SLICE_M * TN;
  static constexpr int RED_BYTES = SPLIT > 1 ? (SPLIT - 1) * SLOT_FLOATS * 4 : 0;
  // bytes a CTA receives from its peers per tile
  static constexpr uint32_t SLICE_TX = (SPLIT - 1) * SLICE_M * TN * 4;
  // swapped split-K: the reduced slice (SLICE_M tokens x 128 weights, bf16)
  // leaves through shared memory with one tensor store
  static constexpr bool RED_TMA = SWAP && SPLIT > 1;
  static constexpr int RSTG_BYTES = RED_TMA ? SLICE_M * 128 * 2 : 0;
  // Thin (swapped) shapes are short launches: once the producer has issued
  // its last load, the next kernel of the stream may launch, so that its
  // prologue overlaps this kernel's reduction and epilogue.
  static constexpr bool EARLY_TRIGGER = SWAP;
  static_assert(SPLIT == 1 || (BT % SPLIT == 0 && SLICE_M % 4 == 0 && COLS % 4 == 0),
                "16-byte pushes of 4 consecutive tokens");
  static_assert(SPLIT == 1 || WPQ == 1, "split-K: a thread holds all tokens of its weight row");
  // on a CTA's last tile the outgoing partials are staged in the idle ring
  static_assert(RED_BYTES <= STAGES * (STAGE_A + STAGE_B), "send staging fits in the ring");
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * STAGE_A;
  static constexpr int OFF_SA = OFF_B + STAGES * STAGE_B;
  // normal-form epilogue staging: each promotion warp owns a bf16 image of
  // its 32 rows x COLS columns, as COLS / 64 tensor-store boxes of 32 rows x
  // 64 columns (128 bytes) in the 128-byte swizzled layout, so the whole
  // slice is written in one pass and leaves with COLS / 64 stores
  static constexpr bool EPI_TMA = !SWAP && SPLIT == 1;
  static constexpr int EPI_BOX = 32 * 128;  // bytes of one box
  static constexpr int EPI_WARP = (COLS / 64) * EPI_BOX;
  static constexpr int EPI_BYTES = EPI_TMA ? PW * EPI_WARP : 0;
  static_assert(!EPI_TMA || COLS % 64 == 0, "epilogue boxes of 64 columns");
  static constexpr int OFF_EPI = EPI_TMA ? (OFF_SA + SAS * STAGE_SA + 1023) / 1024 * 1024
                                        : OFF_SA + SAS * STAGE_SA;
  static constexpr int OFF_RED = OFF_EPI + EPI_BYTES;
  static constexpr int OFF_RSTG = OFF_RED + RED_BYTES;  // 128-byte aligned (RED_BYTES is)
  static constexpr int OFF_BAR = OFF_RSTG + RSTG_BYTES;
  static constexpr int NUM_BARS = 2 * STAGES + 2 * SAS + 4 + 3;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_TABLE = (OFF_MISC + 16 + 15) / 16 * 16;
  // the tile table exists for the grouped forms only; + alignment slack
  static constexpr int table_bytes(int form) { return form == kFormDense ? 0 : kTableMax * 4; }
  static constexpr int smem_bytes(int form) { return OFF_TABLE + table_bytes(form) + 1024; }

  static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "swizzle atoms");
  static_assert(SA_BYTES % 16 == 0, "TMA box inner extent");
  static_assert(!EPI_TMA || OFF_EPI % 1024 == 0, "swizzled tensor-store sources");
  static_assert(!RED_TMA || (OFF_RSTG % 128 == 0 && RSTG_BYTES % 16 == 0), "tensor-store source");
  static_assert(smem_bytes(kFormDense) <= 232448, "shared memory per CTA");
};

struct Tile {
  int valid;
  int e;      // expert (0 for dense)
  int mt;     // token tile within the slab
  int nt;     // weight tile
  int kb0;    // first K block (block-scaled kernel; K-grouped: the expert's first token block)
  int nkb;    // K blocks of the tile
  int phase;  // one-kernel expert FFN: 0 = first GEMM (+ SwiGLU, requant), 1 = second GEMM
  int owned;  // one-kernel expert FFN: the token tile's rows belong to this tile's expert
};

template <class C, int FORM>
__device__ __forceinline__ int total_tiles(const GemmParams& p, const int* table) {
  if (FORM == kFormMasked) return table[p.G];
  if (C::PAIR) return (p.num_mt + 1) / 2 * p.num_nt;  // tiles of two token tiles
  return p.num_mt * p.num_nt;
}

// Tile t of this CTA. With pair MMA the two CTAs of a cluster walk the same
// pair tiles; CTA `pair_rank` owns token tile 2 * (t / num_nt) + pair_rank
// (which may lie past M: it still takes part in the MMAs and stores nothing).
template <class C, int FORM>
__device__ __forceinline__ Tile resolve_tile(const GemmParams& p, const int* table, int t,
                                             int pair_rank) {
  Tile w;
  if (C::PAIR) {
    w.mt = 2 * (t / p.num_nt) + pair_rank;
    w.nt = t % p.num_nt;
    w.e = 0;
    w.valid = 1;
  } else if (FORM == kFormMasked) {
    int lo = 0, hi = p.G;  // table[lo] <= t < table[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (table[mid] <= t) lo = mid; else hi = mid;
    }
    const int local = t - table[lo];
    w.e = lo;
    w.mt = local / p.num_nt;
    w.nt = local % p.num_nt;
    w.valid = 1;
  } else {
    w.mt = t / p.num_nt;
    w.nt = t % p.num_nt;
    if (FORM == kFormContig) {
      w.e = table[w.mt];
      w.valid = w.e >= 0;
    } else {
      w.e = 0;
      w.valid = 1;
    }
  }
  return w;
}

// Runs on warp 0 before the main loops. Contiguous: expert of every token tile
// (read from the tile's first row), -1 for padding tiles. Masked: exclusive
// prefix over experts of the number of (token tile, weight tile) pairs.
template <class C, int FORM>
__device__ void build_table(const GemmParams& p, int* table, int lane) {
  if (FORM == kFormContig) {
    for (int mt = lane; mt < p.num_mt; mt += 32) {
      int v = __ldg(p.m_indices + static_cast<int64_t>(mt) * C::BT);
      if (v >= p.G) {
        raise_status(p.status, 3 /* FG_DEVICE_BAD_M_INDEX */);
        v = -1;
      }
      table[mt] = v < 0 ? -1 : v;
    }
  } else if (FORM == kFormMasked) {
    const int per = (p.G + 31) / 32;
    const int e0 = lane * per;
    const int e1 = min(p.G, e0 + per);
    int local = 0;
    for (int e = e0; e < e1; ++e) {
      int mm = __ldg(p.masked_m + e);
      if (mm < 0 || mm > p.M) {
        raise_status(p.status, 2 /* FG_DEVICE_BAD_MASKED_M */);
        mm = mm < 0 ? 0 : p.M;
      }
      const int cnt = (mm + C::BT - 1) / C::BT * p.num_nt;
      table[e + 1] = cnt;
      local += cnt;
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - local;
    for (int e = e0; e < e1; ++e) {
      run += table[e + 1];
      table[e + 1] = run;
    }
    if (lane == 0) table[0] = 0;
  }
}

// Bounded wait used while tearing down: ignores the abort flag, only the
// time limit, so that copies and MMAs already in flight land before the CTA
// releases its shared and tensor memory.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = wait_clock();
  while (!mbar_try_wait(bar, parity)) {
    if (wait_clock() - t0 > wait_cycles(limit_ns)) return;
  }
}

// Stores `NCOL` consecutive accumulator columns of one tile row (TMEM lane)
// to D. Normal form: the row is a token, the columns weights (16-byte
// vectors). Swapped form: the row is a weight, the columns tokens (2-byte
// stores; the 32 lanes of a warp write 32 consecutive weights of one token).
template <class C, int FORM, int NCOL>
__device__ __forceinline__ void store_tile_part(const GemmParams& p, const Tile& w, int row,
                                                int col0, const float* v, int m_valid,
                                                int row_mi) {
  const int64_t slab = FORM == kFormMasked ? static_cast<int64_t>(w.e) * p.M : 0;
  if (!C::SWAP) {
    const int m = w.mt * C::BT + row;
    bool ok = m < m_valid;
    if (FORM == kFormContig) ok = ok && row_mi >= 0;
    if (!ok) return;
    uint16_t* dst = p.D + (slab + m) * p.N;
#pragma unroll
    for (int j = 0; j < NCOL; j += 8) {
      const int n = w.nt * C::BW + col0 + j;
      if (n < p.N) {
        uint4 q;
        q.x = pack_bf16x2(v[j + 0], v[j + 1]);
        q.y = pack_bf16x2(v[j + 2], v[j + 3]);
        q.z = pack_bf16x2(v[j + 4], v[j + 5]);
        q.w = pack_bf16x2(v[j + 6], v[j + 7]);
        *reinterpret_cast<uint4*>(dst + n) = q;
      }
    }
  } else {
    const int n = w.nt * 128 + row;
    if (n >= p.N) return;
#pragma unroll
    for (int j = 0; j < NCOL; ++j) {
      const int m = w.mt * C::BT + col0 + j;
      bool ok = m < m_valid;
      if (FORM == kFormContig) ok = ok && __ldg(p.m_indices + (m < p.M ? m : 0)) >= 0;
      if (ok) p.D[(slab + m) * p.N + n] = static_cast<uint16_t>(pack_bf16x2(v[j], 0.0f) & 0xFFFFu);
    }
  }
}

// One producer lane's share of a stage: stream 0 = weight tiles, 1 = token
// tiles, 2 = token scales, for the stage's K blocks kq + j * kb_step
// (j < KPS, those below KB).
template <class C, int FORM>
__device__ __forceinline__ void issue_stage(int stream, const GemmParams& p, const Tile& w, int kq,
                                            int kb_step, uint32_t it, uint8_t* sA, uint8_t* sB,
                                            uint8_t* sSA, uint64_t* full, uint64_t* sa_full,
                                            const CUtensorMap* tmA, const CUtensorMap* tmB,
                                            const CUtensorMap* tmSA, int pair_rank) {
  const int s = it % C::STAGES;
  const int q = it % C::SAS;
  int nvalid = 0;
#pragma unroll
  for (int j = 0; j < C::KPS; ++j) nvalid += kq + j * kb_step < p.KB ? 1 : 0;
  if constexpr (C::PAIR) {
    // operand stages of both CTAs complete on the leader's barrier, which
    // expects the bytes of both
    if (stream < 2) {
      const uint32_t leader_full = mapa_shared(smem_u32(&full[s]), 0);
      if (stream == 0) {
        if (pair_rank == 0) mbar_arrive_expect_tx(&full[s], 2 * C::B_BYTES);
        tma_load_2d_pair(sB + s * C::STAGE_B, tmB, leader_full, kq * 128,
                         w.e * p.N + w.nt * C::BW + pair_rank * C::B_ROWS);
      } else {
        if (pair_rank == 0) mbar_arrive_expect_tx(&full[s], 2 * C::A_BYTES);
        tma_load_2d_pair(sA + s * C::STAGE_A, tmA, leader_full, kq * 128, w.mt * C::BT);
      }
      return;
    }
  }
  if (stream == 0) {
    mbar_arrive_expect_tx(&full[s], nvalid * C::B_BYTES);
    for (int j = 0; j < nvalid; ++j)
      tma_load_2d(sB + s * C::STAGE_B + j * C::B_BYTES, tmB, &full[s], (kq + j * kb_step) * 128,
                  w.e * p.N + w.nt * C::BW);
  } else if (stream == 1) {
    mbar_arrive_expect_tx(&full[s], nvalid * C::A_BYTES);
    for (int j = 0; j < nvalid; ++j)
      tma_load_2d(sA + s * C::STAGE_A + j * C::A_BYTES, tmA, &full[s], (kq + j * kb_step) * 128,
                  (FORM == kFormMasked ? w.e * p.M : 0) + w.mt * C::BT);
  } else {
    mbar_arrive_expect_tx(&sa_full[q], nvalid * C::SA_BYTES);
    for (int j = 0; j < nvalid; ++j)
      tma_load_2d(sSA + q * C::STAGE_SA + j * C::SA_STAGE, tmSA, &sa_full[q], w.mt * C::BT,
                  (FORM == kFormMasked ? w.e * p.KB : 0) + kq + j * kb_step);
  }
}

template <class C, int FORM>
__global__ void __launch_bounds__(C::NUM_THREADS, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmD,
                    const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem + C::OFF_A;
  uint8_t* sB = smem + C::OFF_B;
  uint8_t* sSA = smem + C::OFF_SA;
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + C::STAGES;
  uint64_t* sa_full = empty + C::STAGES;   // token scales of a stage have landed
  uint64_t* sa_empty = sa_full + C::SAS;   // ... and have been read by the promotion warps
  uint64_t* tfull = sa_empty + C::SAS;
  uint64_t* tempty = tfull + 2;
  uint64_t* red_ready = tempty + 2;    // all partials of the current tile are in place
  uint64_t* red_free = red_ready + 1;  // every CTA has finished reading them
  uint64_t* grp = red_free + 1;        // all promotion warps of this CTA (bounded group sync)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  int* table = reinterpret_cast<int*>(smem + C::OFF_TABLE);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // tiles are dealt to CTAs (or, with split-K, to clusters) round robin;
  // the K blocks of a tile to the CTAs of its cluster
  static_assert(!C::PAIR || FORM == kFormDense, "pair MMA covers the dense form");
  const int t_first = C::CLUSTER > 1 ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
  const int t_step = C::CLUSTER > 1 ? static_cast<int>(num_clusters_x()) : static_cast<int>(gridDim.x);
  const int kb_first = C::SPLIT > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  const int pair_rank = C::PAIR ? static_cast<int>(cluster_ctarank()) : 0;
  constexpr int kb_step = C::SPLIT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 2);               // weight- and token-tile lanes' expect_tx
      mbar_init(&empty[s], 1);              // the MMA commit
    }
    for (int q = 0; q < C::SAS; ++q) {
      mbar_init(&sa_full[q], 1);            // the scale lane's expect_tx
      mbar_init(&sa_empty[q], C::PW);       // one arrival per promotion warp
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], C::PAIR ? 2 * C::PW : C::PW);  // pair: the leader's counts both CTAs
    }
    mbar_init(red_ready, 1);                 // own expect_tx; peers' bytes complete_tx
    mbar_init(red_free, C::SPLIT * C::PW);   // one arrival per promotion warp of each CTA
    mbar_init(grp, C::PW);                   // one arrival per promotion warp
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmSA);
    if (C::EPI_TMA || C::RED_TMA) tma_prefetch_desc(&tmD);
  }
  if constexpr (!C::PAIR) {
    if (warp == 1) {
      tmem_alloc(tmem_slot, C::TMEM_COLS);
      tmem_relinquish();
    }
  }
  // Peers address this CTA's barriers only after the cluster barrier
  // completes (its wait comes after the CTA-wide barrier below).
  __syncwarp();
  if constexpr (C::CLUSTER > 1) cluster_arrive_relaxed();
  // Everything above may overlap the previous kernel; memory comes after this.
  grid_dependency_wait();
  if (warp == 0) build_table<C, FORM>(p, table, lane);
  tc_fence_before();
  __syncwarp();
  __syncthreads();
  if constexpr (C::CLUSTER > 1) cluster_wait();  // peers' barriers are initialised
  if constexpr (C::PAIR) {
    // the pair's tensor memory, allocated jointly once both CTAs run
    if (warp == 1) {
      tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
      tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
  }
  tc_fence_after();

  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.status, p.timeout_ns};
  const int total = total_tiles<C, FORM>(p, table);

  if (warp < C::PW_BASE) {
  if constexpr (C::REG_SPLIT) warpgroup_reg_dealloc<C::REG_LOW>();
  // Producer streams: 0 = weight tiles, 1 = token tiles, 2 = token scales.
  // With 8 promotion warps each stream has a warp of its own (warps 0, 2 and
  // 3), so that one stream's barrier wait does not hold up the others (three
  // lanes of one warp diverge, and a waiting lane stalls its warp); with 4
  // they are lanes 0..2 of warp 0.
  constexpr bool OWN_WARPS = C::PW_BASE == 4;
  const int stream = OWN_WARPS ? (warp == 0 ? 0 : warp - 1) : lane;
  if (warp != 1) {
    // ------------------------------------------------------------ producer
    if (OWN_WARPS ? lane == 0 : (warp == 0 && lane < 3)) {
      uint32_t it = 0;
      for (int t = t_first; t < total; t += t_step) {
        const Tile w = resolve_tile<C, FORM>(p, table, t, pair_rank);
        if (!w.valid) continue;
        for (int kq = kb_first; kq < p.KB; kq += C::KPS * kb_step, ++it) {
          if (stream < 2) {
            const int s = it % C::STAGES;
            if (!mbar_wait(&empty[s], ((it / C::STAGES) & 1u) ^ 1u, ctl)) goto producer_done;
          } else {
            const int q = it % C::SAS;
            if (!mbar_wait(&sa_empty[q], ((it / C::SAS) & 1u) ^ 1u, ctl)) goto producer_done;
          }
          issue_stage<C, FORM>(stream, p, w, kq, kb_step, it, sA, sB, sSA, full, sa_full, &tmA, &tmB,
                               &tmSA, pair_rank);
        }
      }
      // every load of this CTA is issued: the next kernel of the stream may
      // launch (it waits for this grid's completion before touching memory)
      if (C::EARLY_TRIGGER) grid_launch_dependents();
    producer_done:
      // Before the CTA exits, the last fill of every stage must have landed
      // and been released (its TMA bytes and the MMA commit's arrival).
      if (stream == 0) {
        for (uint32_t s = 0; s < C::STAGES && s < it; ++s) {
          const uint32_t last = (it - 1 - s) / C::STAGES * C::STAGES + s;
          // (a pair's operand bytes complete on the leader's barrier)
          if (!C::PAIR || pair_rank == 0) drain_wait(&full[s], (last / C::STAGES) & 1u, kDrainLimitNs);
          drain_wait(&empty[s], (last / C::STAGES) & 1u, kDrainLimitNs);
        }
      } else if (stream == 2) {
        for (uint32_t q = 0; q < C::SAS && q < it; ++q) {
          const uint32_t last = (it - 1 - q) / C::SAS * C::SAS + q;
          drain_wait(&sa_full[q], (last / C::SAS) & 1u, kDrainLimitNs);
          drain_wait(&sa_empty[q], (last / C::SAS) & 1u, kDrainLimitNs);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (converged: descriptors stay
    // warp-uniform, which keeps each tcgen05 issue short); one elected lane
    // issues the MMAs and commits.
    if (pair_rank == 0) {  // a pair's MMAs are issued by its leader
      constexpr uint32_t idesc = mma_idesc_e4m3(C::MMA_M, C::MMA_N);
      uint32_t it = 0;
      // the next iteration's TMEM buffer / operand stage were seen free /
      // full by a non-blocking peek made while this iteration's MMAs ran
      bool empty_seen = false, full_seen = false;
      for (int t = t_first; t < total; t += t_step) {
        const Tile w = resolve_tile<C, FORM>(p, table, t, pair_rank);
        if (!w.valid) continue;
        for (int kq = kb_first; kq < p.KB; kq += C::KPS * kb_step, ++it) {
          const int s = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1u;
          const int b = it & 1;
          const uint32_t tph = (it >> 1) & 1u;
          if (!empty_seen && !warp_wait(&tempty[b], tph ^ 1u, ctl, lane)) goto mma_done;
          tc_fence_after();
          if (!full_seen && !warp_wait(&full[s], ph, ctl, lane)) goto mma_done;
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int j = 0; j < C::KPS; ++j) {
              if (kq + j * kb_step >= p.KB) break;
              const uint8_t* a_tile = sA + s * C::STAGE_A + j * C::A_BYTES;
              const uint8_t* b_tile = sB + s * C::STAGE_B + j * C::B_BYTES;
              const uint64_t adesc = smem_desc_sw128(smem_u32(C::SWAP ? b_tile : a_tile));
              const uint64_t bdesc = smem_desc_sw128(smem_u32(C::SWAP ? a_tile : b_tile));
              // one fresh partial per K block: slot (b, j) of tensor memory
              const uint32_t d = tmem_base + static_cast<uint32_t>((b * C::KPS + j) * C::MMA_N);
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                // advance 32 bytes (= 32 e4m3 along K) inside the 128-byte swizzled row
                if constexpr (C::PAIR)
                  mma_f8_pair(d, adesc + 2 * k, bdesc + 2 * k, idesc, k > 0 ? 1u : 0u);
                else
                  mma_f8(d, adesc + 2 * k, bdesc + 2 * k, idesc, k > 0 ? 1u : 0u);
              }
            }
            if constexpr (C::PAIR) {
              mma_commit_pair(&empty[s]);  // both CTAs' stage s and TMEM buffer b
              mma_commit_pair(&tfull[b]);
            } else {
              mma_commit(&empty[s]);
              mma_commit(&tfull[b]);
            }
          }
          {
            // peek at the next iteration's buffer and stage while these MMAs
            // run: a phase seen complete here needs no blocking wait (phases
            // of both barriers advance at most one ahead of this warp)
            const uint32_t nx = it + 1;
            empty_seen = __all_sync(0xffffffffu, mbar_test_wait(&tempty[nx & 1], ((nx >> 1) & 1u) ^ 1u));
            full_seen = __all_sync(0xffffffffu, mbar_test_wait(&full[nx % C::STAGES], (nx / C::STAGES) & 1u));
          }
        }
      }
    mma_done:
      if (it > 0 && lane == 0) drain_wait(&tfull[(it - 1) & 1], ((it - 1) >> 1) & 1u, kDrainLimitNs);
    }
  }
  } else {
    // ------------------------------------------------------------ promotion + epilogue
    if constexpr (C::REG_SPLIT) warpgroup_reg_alloc<C::REG_HIGH>();
    const int pw = warp - C::PW_BASE;
    const int quad = warp & 3;          // TMEM lanes this warp may access
    const int part = pw >> 2;           // column slice of the accumulator
    const int row = quad * 32 + lane;   // TMEM lane = row of the lane operand
    const int c0 = part * C::COLS;
    const uint32_t t_lane = static_cast<uint32_t>(quad * 32) << 16;
    uint32_t it = 0;
    uint32_t tiles_done = 0;
    uint32_t grp_phase = 0;   // uses of the promotion group barrier
    for (int t = t_first; t < total; t += t_step) {
      const Tile w = resolve_tile<C, FORM>(p, table, t, pair_rank);
      if (!w.valid) continue;
      // row bounds of this tile's token slab (read early, used in the epilogue)
      int m_valid = p.M;
      if (FORM == kFormMasked) {
        m_valid = __ldg(p.masked_m + w.e);
        m_valid = m_valid < 0 ? 0 : (m_valid > p.M ? p.M : m_valid);
      }
      // weight scale of this thread's 128 weight rows: one per K block, read
      // from global memory one stage ahead
      const int nb = w.nt * (C::BW / 128) + (C::SWAP ? 0 : c0 / 128);
      const float* sb_row = p.sfb + (static_cast<int64_t>(w.e) * p.NB + min(nb, p.NB - 1)) * p.KB;
      float sb_next[C::KPS];
#pragma unroll
      for (int j = 0; j < C::KPS; ++j) {
        const int kb = kb_first + j * kb_step;
        sb_next[j] = kb < p.KB ? __ldg(sb_row + kb) : 0.0f;
      }
      float acc[C::COLS];
#pragma unroll
      for (int j = 0; j < C::COLS; ++j) acc[j] = 0.0f;

      for (int kq = kb_first; kq < p.KB; kq += C::KPS * kb_step, ++it) {
        float sbv[C::KPS];
#pragma unroll
        for (int j = 0; j < C::KPS; ++j) {
          sbv[j] = sb_next[j];
          const int kb = kq + (C::KPS + j) * kb_step;
          sb_next[j] = kb < p.KB ? __ldg(sb_row + kb) : 0.0f;
        }
        const int q = it % C::SAS;
        const int b = it & 1;
        const uint32_t tph = (it >> 1) & 1u;
        if (!mbar_wait(&sa_full[q], (it / C::SAS) & 1u, ctl)) goto promo_done;
        if (!mbar_wait(&tfull[b], tph, ctl)) goto promo_done;
        tc_fence_after();
        if constexpr (!C::SWAP && C::KPS == 1 && C::COLS % 64 == 0) {
          // normal form: the thread's columns in batches of 64 (two 32-column
          // TMEM loads, one wait); the TMEM buffer and the scale slot are
          // released as soon as the last batch is in registers, before it is
          // folded in with packed fused multiply-adds
          const float* sa_s = reinterpret_cast<const float*>(sSA + q * C::STAGE_SA);
          const float scale = sa_s[row] * sbv[0];
          const uint32_t taddr = tmem_base + t_lane + static_cast<uint32_t>(b * C::MMA_N + c0);
#pragma unroll
          for (int h = 0; h < C::COLS / 64; ++h) {
            uint32_t r0[32], r1[32];
            tmem_ld32_issue(taddr + 64 * h, r0);
            tmem_ld32_issue(taddr + 64 * h + 32, r1);
            tmem_wait_ld64(r0, r1);
            if (h == C::COLS / 64 - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) {
                if constexpr (C::PAIR)  // the leader's MMA waits for both CTAs
                  mbar_arrive_remote(mapa_shared(smem_u32(&tempty[b]), 0));
                else
                  mbar_arrive(&tempty[b]);
                mbar_arrive(&sa_empty[q]);
              }
            }
            float* a = acc + 64 * h;
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              fma2(a[j], a[j + 1], __uint_as_float(r0[j]), __uint_as_float(r0[j + 1]), scale);
              fma2(a[32 + j], a[33 + j], __uint_as_float(r1[j]), __uint_as_float(r1[j + 1]), scale);
            }
          }
        } else {
#pragma unroll
        for (int jk = 0; jk < C::KPS; ++jk) {
          if (kq + jk * kb_step >= p.KB) break;
          const float* sa_s = reinterpret_cast<const float*>(sSA + q * C::STAGE_SA + jk * C::SA_STAGE);
          const uint32_t taddr = tmem_base + t_lane +
                                 static_cast<uint32_t>((b * C::KPS + jk) * C::MMA_N + c0);
          if (!C::SWAP) {
            const float scale = sa_s[row] * sbv[jk];
#pragma unroll
            for (int ch = 0; ch < C::COLS; ch += (C::COLS - ch >= 64 && C::COLS <= 64 ? 64 : 32)) {
              if (C::COLS - ch >= 64 && C::COLS <= 64) {
                float v[64];
                tmem_ld64(taddr + ch, v);
#pragma unroll
                for (int j = 0; j < 64; ++j) acc[ch + j] = fmaf(v[j], scale, acc[ch + j]);
              } else if (C::COLS - ch >= 32) {
                float v[32];
                tmem_ld32(taddr + ch, v);
#pragma unroll
                for (int j = 0; j < 32; ++j) acc[ch + j] = fmaf(v[j], scale, acc[ch + j]);
                if (C::COLS > 64) pin_regs<32>(acc + ch);
              } else if (C::COLS - ch >= 16) {
                float v[16];
                tmem_ld16(taddr + ch, v);
#pragma unroll
                for (int j = 0; j < 16; ++j) acc[ch + j] = fmaf(v[j], scale, acc[ch + j]);
              }
            }
          } else {
            const float sbs = sbv[jk];
#pragma unroll
            for (int ch = 0; ch < C::COLS; ch += (C::COLS - ch >= 64 && C::COLS <= 64 ? 64 : 32)) {
              if (C::COLS - ch >= 64 && C::COLS <= 64) {
                float v[64];
                tmem_ld64(taddr + ch, v);
#pragma unroll
                for (int j = 0; j < 64; ++j)
                  acc[ch + j] = fmaf(v[j], sbs * sa_s[c0 + ch + j], acc[ch + j]);
              } else if (C::COLS - ch >= 32) {
                float v[32];
                tmem_ld32(taddr + ch, v);
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  acc[ch + j] = fmaf(v[j], sbs * sa_s[c0 + ch + j], acc[ch + j]);
              } else if (C::COLS - ch >= 16) {
                float v[16];
                tmem_ld16(taddr + ch, v);
#pragma unroll
                for (int j = 0; j < 16; ++j)
                  acc[ch + j] = fmaf(v[j], sbs * sa_s[c0 + ch + j], acc[ch + j]);
              } else {
                float v[8];
                tmem_ld8(taddr + ch, v);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                  acc[ch + j] = fmaf(v[j], sbs * sa_s[c0 + ch + j], acc[ch + j]);
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (C::PAIR)
            mbar_arrive_remote(mapa_shared(smem_u32(&tempty[b]), 0));
          else
            mbar_arrive(&tempty[b]);
          mbar_arrive(&sa_empty[q]);
        }
        }
      }

      // -------------------------------------------------------- epilogue
      if constexpr (C::SPLIT == 1) {
        int row_mi = 0;
        if (FORM == kFormContig && !C::SWAP) {
          const int m = w.mt * C::BT + row;
          row_mi = m < p.M ? __ldg(p.m_indices + m) : -1;
        }
        bool staged = false;
        if constexpr (C::EPI_TMA) {
          const int m = w.mt * C::BT + row;
          const bool ok = m < m_valid && (FORM != kFormContig || row_mi >= 0);
          if (__all_sync(0xffffffffu, ok)) {
            staged = true;
            // D rows of this warp: the slab row of its first token
            const int y = (FORM == kFormMasked ? w.e * p.M : 0) + w.mt * C::BT + quad * 32;
            uint8_t* img = smem + C::OFF_EPI + pw * C::EPI_WARP;
            // the stores of this warp's previous tile have read the image
            if (lane == 0) bulk_wait_group_read<0>();
            __syncwarp();
            // row `lane` of box h: 16-byte chunk c (columns h*64 + 8c ..) at
            // chunk position c ^ (lane % 8), the tensor map's 128-byte swizzle
#pragma unroll
            for (int h = 0; h < C::COLS / 64; ++h) {
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                const float* v = acc + h * 64 + c * 8;
                *reinterpret_cast<uint4*>(img + h * C::EPI_BOX + lane * 128 + ((c ^ (lane & 7)) * 16)) =
                    make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                               pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
              }
            }
            fence_proxy_async_shared();
            __syncwarp();
            if (lane == 0) {
#pragma unroll
              for (int h = 0; h < C::COLS / 64; ++h) {
                const int x = w.nt * C::BW + c0 + h * 64;
                if (x < p.N) tma_store_2d(&tmD, img + h * C::EPI_BOX, x, y);  // columns past N clipped
              }
              bulk_commit_group();
            }
          }
        }
        if (!staged) store_tile_part<C, FORM, C::COLS>(p, w, row, c0, acc, m_valid, row_mi);
      } else {
        const uint32_t red_addr = smem_u32(red);
        const uint32_t ready_addr = smem_u32(red_ready);
        const int rank = kb_first;
        // (1) the receivers must have read the previous tile's slots
        if (tiles_done > 0 &&
            !mbar_wait_cluster(red_free, (tiles_done - 1) & 1u, abort_flag, p.status, p.timeout_ns))
          goto promo_done;
        // (2) expect this tile's bytes from every peer
        if (threadIdx.x == C::PW_BASE * 32) mbar_arrive_expect_tx(red_ready, C::SLICE_TX);
        // (3) push the partial values of the tokens other CTAs own (token m
        //     belongs to CTA m / SLICE_M) into their slot for this CTA; this
        //     thread's lane is weight `row`, its columns tokens c0 .. c0 + COLS
        if (t + t_step >= total) {
          // last tile of this CTA: the ring is idle (the tile's last MMA has
          // completed and no load follows), so each peer's slot image is
          // assembled there and sent with one bulk copy
          float* images = reinterpret_cast<float*>(smem + C::OFF_A);
#pragma unroll
          for (int j = 0; j < C::COLS; j += 4) {
            const int m = c0 + j;
            const int dst = m / C::SLICE_M;
            if (dst != rank) {
              float* img = images + (dst < rank ? dst : dst - 1) * C::SLOT_FLOATS;
              *reinterpret_cast<float4*>(img + ((m % C::SLICE_M) / 4 * C::TN + row) * 4) =
                  make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
            }
          }
          fence_proxy_async_shared();
          __syncwarp();
          if (lane == 0) mbar_arrive(grp);
          if (!mbar_wait(grp, grp_phase++ & 1u, ctl)) goto promo_done;
          if (threadIdx.x == C::PW_BASE * 32) {
            for (int dst = 0; dst < C::SPLIT; ++dst) {
              if (dst == rank) continue;
              const uint32_t off = static_cast<uint32_t>((rank < dst ? rank : rank - 1) * C::SLOT_FLOATS * 4);
              bulk_copy_to_cluster(mapa_shared(red_addr + off, static_cast<uint32_t>(dst)),
                                   images + (dst < rank ? dst : dst - 1) * C::SLOT_FLOATS,
                                   C::SLOT_FLOATS * 4, mapa_shared(ready_addr, static_cast<uint32_t>(dst)));
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < C::COLS; j += 4) {
            const int m = c0 + j;
            const int dst = m / C::SLICE_M;
            if (dst != rank) {
              const int slot = rank < dst ? rank : rank - 1;
              const uint32_t off = static_cast<uint32_t>(
                  (slot * C::SLOT_FLOATS + ((m % C::SLICE_M) / 4 * C::TN + row) * 4) * 4);
              st_async_f4(mapa_shared(red_addr + off, static_cast<uint32_t>(dst)),
                          make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]),
                          mapa_shared(ready_addr, static_cast<uint32_t>(dst)));
            }
          }
        }
        // (4) wait until every peer's bytes for this CTA's tokens have landed
        if (!mbar_wait_cluster(red_ready, tiles_done & 1u, abort_flag, p.status, p.timeout_ns))
          goto promo_done;
        {
          const bool more = t + t_step < total;  // will peers push into these slots again?
          // (5) weight `row`: sum its SLICE_M owned tokens over the CTAs in
          //     split order (its own values from registers), so the result does
          //     not depend on which CTA finished first
          float sum[C::SLICE_M];
#pragma unroll
          for (int j = 0; j < C::SLICE_M; ++j) sum[j] = 0.0f;
#pragma unroll
          for (int r = 0; r < C::SPLIT; ++r) {
            if (r == rank) {
#pragma unroll
              for (int j = 0; j < C::SLICE_M; ++j) sum[j] += acc[r * C::SLICE_M + j];
            } else {
              const float* src = red + (r < rank ? r : r - 1) * C::SLOT_FLOATS + row * 4;
#pragma unroll
              for (int j = 0; j < C::SLICE_M; j += 4) {
                const float4 v = *reinterpret_cast<const float4*>(src + j * C::TN);
                sum[j] += v.x;
                sum[j + 1] += v.y;
                sum[j + 2] += v.z;
                sum[j + 3] += v.w;
              }
            }
          }
          if (more) {
            __syncwarp();
            if (lane == 0)
              for (int r = 0; r < C::SPLIT; ++r) mbar_arrive_cluster(mapa_shared(smem_u32(red_free), r));
          }
          if constexpr (C::RED_TMA && FORM == kFormDense) {
            // bf16 slice [SLICE_M tokens][128 weights] in shared memory, then
            // one tensor store (rows past M and columns past N are clipped)
            const int y = w.mt * C::BT + rank * C::SLICE_M;
            uint16_t* stg = reinterpret_cast<uint16_t*>(smem + C::OFF_RSTG);
            // the previous tile's store has finished reading the buffer: its
            // issuing thread waits for that before this group barrier
            if (tiles_done > 0) {
              if (threadIdx.x == C::PW_BASE * 32) bulk_wait_group_read<0>();
              __syncwarp();
              if (lane == 0) mbar_arrive(grp);
              if (!mbar_wait(grp, grp_phase++ & 1u, ctl)) goto promo_done;
            }
#pragma unroll
            for (int j = 0; j < C::SLICE_M; ++j)
              stg[j * 128 + row] = static_cast<uint16_t>(pack_bf16x2(sum[j], 0.0f) & 0xFFFFu);
            fence_proxy_async_shared();
            __syncwarp();
            if (lane == 0) mbar_arrive(grp);
            if (!mbar_wait(grp, grp_phase++ & 1u, ctl)) goto promo_done;
            if (threadIdx.x == C::PW_BASE * 32 && y < m_valid) {
              tma_store_2d(&tmD, stg, w.nt * 128, y);
              bulk_commit_group();
            }
          } else {
            store_tile_part<C, FORM, C::SLICE_M>(p, w, row, rank * C::SLICE_M, sum, m_valid, 0);
          }
        }
        ++tiles_done;
      }
    }
  promo_done:
    // tensor stores of the epilogue have completed (global writes done,
    // shared memory no longer read)
    // this warp's tensor stores have finished reading shared memory
    if ((C::EPI_TMA || C::RED_TMA) && lane == 0) bulk_wait_group_read<0>();
  }

  // ---------------------------------------------------------------- teardown
  // Single lanes of warpgroup 0 ran their roles alone: reconverge every warp
  // before the CTA-wide barrier (a barrier reached by part of a warp does not
  // wait for the rest of the CTA).
  __syncwarp();
  tc_fence_before();
  // No CTA may leave while a peer can still write its shared memory; the
  // cluster barrier covers every thread of the CTA as well.
  if constexpr (C::CLUSTER > 1) {
    // every CTA arrives only after all bytes sent to it have landed (split-K)
    // or all MMAs writing its tensor memory have completed (pair), so when
    // the barrier completes no transfer reads or writes any CTA's memory
    cluster_arrive_relaxed();
    cluster_wait();
  } else {
    __syncthreads();
  }
  grid_launch_dependents();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (C::PAIR) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    else tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace fg
