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
// Scale words: the block-scaled MMA reads, per row, a 32-bit word from tensor
// memory and uses the byte its scale-factor id selects. One word carries the
// scales of four consecutive 128-wide K blocks (byte k = K block 4q + k), so
// the scale groups are converted and copied to tensor memory once per four K
// blocks (a "quad"), through their own ring of SFS slots.
//
// The MMA-issuing thread is the critical resource: on sm_100a each tcgen05
// instruction occupies it for tens of cycles, so everything else it does per
// K block (barrier waits, scale copies, commits, bookkeeping) directly idles
// the tensor pipe. Hence quads, KPS K blocks per pipeline stage (one wait and
// one commit per stage) and a non-blocking peek at the next stage's barrier
// while the current stage's MMAs are being issued.
//
// CTA roles (one CTA per SM, persistent over 128-token x BW-weight tiles):
//   warp 0      producer: lane 0 loads the weight tiles, lane 1 the token
//               tiles of each stage's K blocks onto its "full" barrier (TMA);
//               lane 2 the fp32 scales of each quad onto its "sa full"
//               barrier: the 128 x 4 token scales with one TMA copy, the (at
//               most three per K block) weight-block scales the tile's rows
//               touch with 4-byte cp.async copies.
//   warp 1      MMA issuer (converged warp, one elected lane issues): per
//               quad, waits for its scale groups and copies
//               them to tensor memory (tcgen05.cp); per K block 4 block-scaled
//               MMAs (K = 32 each) into the tile's accumulator; commits each
//               stage to "empty", each quad to "sf empty" and each finished
//               accumulator to "tmem full".
//   warp 2      scale converter: per quad takes the staged fp32 scales,
//               keeps their exponent bytes (UE8M0 has the fp32 exponent's
//               bias), packs four K blocks per word in the shared layout
//               tcgen05.cp expects and arrives on the slot's "sf full".
//   warp 3      idle (keeps the epilogue warps aligned to TMEM lane quadrants)
//   warps 4..   epilogue: per tile, 32 accumulator columns at a time from
//               tensor memory to registers, bf16, a 64-byte-swizzled shared
//               image of 32 rows x 32 columns and a tensor store; the
//               accumulator is released as soon as its last columns are read.
// With two accumulators (BW <= 224) the epilogue of one tile overlaps the
// MMAs of the next; with BW = 256 the MMAs wait for the accumulator to be
// read (8 epilogue warps keep that short).
//
// Pair form (PAIR): the two CTAs of a cluster compute one tile of 256 tokens
// x BW weights with tcgen05 cta_group::2. Dense: token tiles 2j and 2j + 1.
// Masked: consecutive token tiles of one expert's slab. Contiguous: a "pair
// unit" table built by warp 0 pairs consecutive token tiles within each run
// of tiles of one expert; a run of odd length ends with a unit whose second
// tile belongs to no row of that expert (it still loads its half of the
// weight tile, which the leader's MMAs need, and stores nothing). Each CTA loads its 128
// token rows and half of the weight rows. The block-scaled pair MMA reads, in
// each CTA's tensor memory, the scales of that CTA's token rows and of all BW
// weight rows, so both CTAs stage and convert the weight scales of the whole
// tile. The leader (rank 0) issues the copies, MMAs and commits, which arrive
// on both CTAs' barriers; operand bytes of both CTAs complete on the leader's
// "full" barrier; the peer's converter and epilogue arrive on the leader's
// "sf full" and "tmem empty" barriers through the cluster.
//
// Fused expert-FFN epilogue (EPI = 1, first GEMM of the expert FFN): W1 holds
// I gate rows then I up rows per expert; the tile of weight tile nt is the
// 128 gate rows nt*128.. and the 128 up rows I + nt*128.. (a pair's CTAs load
// one block each), so each token row of the tile holds 128 gate and the
// matching 128 up values. The epilogue rounds them to bf16, computes
// h = bf16(silu(gate) * up) (act.cuh), takes the row's 128-wide amax and its
// power-of-two scale, and writes the e4m3 codes of h and the scale in the
// per-token layout the second GEMM reads (optionally also the bf16 gate and
// up values). The arithmetic is that of per_token_cast_to_fp8_ue8m0.
//
// K-grouped GEMM (EPI = 2, form kFormKGrouped: the weight gradients of the
// experts in FP8 training): the contraction runs over tokens whose expert
// ranges are stacked along K, so a tile (expert e, mt, nt) runs over the K
// blocks of expert e only; both operands carry one scale per row per
// 128-token block (the per-row B scales arrive with a second TMA box beside
// the token scales); the fp32 result goes out through 128-byte-swizzled
// 32 x 32 boxes. An expert without tokens gets zeros (no MMA runs for it).
#pragma once

#include <cstdint>
#include <cuda.h>

#include "act.cuh"
#include "gemm.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace fg {

template <int BW_, int STAGES_, int ACC_, int EPQ_, bool PAIR_, int KPS_, int EPI_ = 0>
struct MxCfg {
  // 0: bf16 D; 1: SwiGLU + UE8M0 requantization; 2: K-grouped, fp32 D;
  // 3: the whole expert FFN in one launch (first-GEMM tiles with the EPI = 1
  // epilogue, then second-GEMM tiles with a bf16 epilogue)
  static constexpr int EPI = EPI_;
  static constexpr bool FFN = EPI == 1 || EPI == 3;  // tiles of 128 gate + 128 up weight rows
  static constexpr bool FUSED = EPI == 3;
  static constexpr int BT = 128;          // token rows per CTA tile
  static constexpr int BW = BW_;          // weight rows per tile (MMA N)
  static constexpr bool SWAP = false;     // tile helpers of gemm.cuh: tokens on the lanes
  static constexpr bool PAIR = PAIR_;
  static constexpr int CLUSTER = PAIR ? 2 : 1;
  static constexpr int MMA_M = PAIR ? 256 : 128;
  static constexpr int B_ROWS = PAIR ? BW / 2 : BW;  // weight rows this CTA loads
  static constexpr int STAGES = STAGES_;
  static constexpr int KPS = KPS_;        // K blocks per pipeline stage
  static_assert(KPS == 1 || KPS == 2 || KPS == 4, "stages tile the 4-block quads");
  static constexpr int ACC = ACC_;        // accumulators in tensor memory
  static constexpr int EPQ = EPQ_;        // epilogue warps per TMEM lane quadrant
  static_assert(BW % 32 == 0 && BW >= 32 && BW <= 256, "tcgen05 N, 32-column chunks");
  static_assert(!PAIR || B_ROWS % 16 == 0, "pair: half tiles of whole 8-row swizzle atoms");
  static_assert(!FFN || (BW == 256 && ACC == 1 && EPQ == 1),
                "fused FFN epilogue: 128 gate + 128 up columns, one accumulator, one warp per quadrant");
  // weight rows per tensor load: the fused FFN tile is two 128-row blocks
  // (the second GEMM's tiles of the one-kernel FFN load 128 consecutive rows
  // per box as well)
  static constexpr int B_BOX = FFN ? 128 : B_ROWS;
  static constexpr int B_LOADS = B_ROWS / B_BOX;
  static constexpr int EW = 4 * EPQ;      // epilogue warps
  static constexpr int ECOLS = BW / EPQ;  // accumulator columns per epilogue warp
  static_assert(ECOLS % 32 == 0, "epilogue chunks of 32 columns");
  static constexpr int EPI_BASE = 4;      // first epilogue warp
  static constexpr int NUM_THREADS = (EPI_BASE + EW) * 32;
  // scale groups of one slot: 128 token rows, ceil(BW / 128) x 128 weight rows
  static constexpr int SFB_GROUPS = (BW + 127) / 128;
  static constexpr int SF_COLS = 4 * (1 + SFB_GROUPS);    // tensor-memory columns per slot
  static constexpr int SF_BYTES = 512 * (1 + SFB_GROUPS);  // shared bytes per slot
  static constexpr int SFS = 3;           // scale slots (quads in flight)
  // staged fp32 scales of a quad: 4 x 128 token scales (one TMA box), then
  // 4 x NBT weight-block scales ([k][j]: K block 4q + k, block nb0 + j)
  // one-kernel FFN: the second GEMM's tiles are BW2 = 224 weight rows wide
  // with two accumulators (the tile's K loop is short, so its epilogue must
  // overlap the next tile's MMAs); tensor memory: the first GEMM's 256-column
  // accumulator at column 0, the second GEMM's two at 0 and BW2, then the
  // scale slots. Staged weight-block scales: 2 for the first GEMM (gate, up),
  // up to 3 for a 224-row tile of the second.
  static constexpr int BW2 = FUSED ? 224 : BW;
  static constexpr int B_ROWS2 = PAIR ? BW2 / 2 : BW2;
  static constexpr int ACCB = FUSED ? 2 : ACC;  // accumulator barrier pairs
  static constexpr int SF_BASE = FUSED ? 2 * BW2 : ACC * BW;
  static_assert(!FUSED || (2 * BW2 >= BW && B_ROWS2 % 16 == 0 && B_ROWS2 <= 256), "second-GEMM tiles");
  static constexpr int NBT = FUSED ? 3 : (FFN ? 2 : SFB_GROUPS + 1);
  static constexpr int RAW_A = 4 * 512;
  // K-grouped: per-row weight scales, BW rows x 4 K blocks (one TMA box)
  static constexpr int RAW_B = EPI == 2 ? 4 * BW * 4 : 128;
  static constexpr int RAW_BYTES = RAW_A + (RAW_B + 127) / 128 * 128;
  static constexpr int RAWS = 2;          // staged-scale ring
  static_assert(EPI == 2 || 4 * NBT * 4 <= RAW_BYTES - RAW_A, "staged weight-block scales");
  static constexpr int TMEM_USED = SF_BASE + SFS * SF_COLS;
  static_assert(TMEM_USED <= 512, "TMEM has 512 columns");
  static constexpr int TMEM_COLS = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64
                                   : TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
  static constexpr int A_BYTES = BT * 128;       // one K block of the token tile
  static constexpr int B_BYTES = B_ROWS * 128;   // one K block of this CTA's weight rows
  static constexpr int STAGE_A = KPS * A_BYTES;
  static constexpr int STAGE_B = KPS * B_BYTES;
  // epilogue image buffers per warp, each one box of 32 rows x 32 columns
  // (bf16: 64-byte rows; fp32: 128-byte rows)
  static constexpr int EPI_RING = EPI == 2 ? 1 : 2;
  static constexpr int BOX_BYTES = EPI == 2 ? 32 * 128 : 32 * 64;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * STAGE_A;
  static constexpr int OFF_SF = OFF_B + STAGES * STAGE_B;
  static constexpr int OFF_RAW = OFF_SF + SFS * SF_BYTES;  // 128-byte aligned
  static constexpr int OFF_EPI = (OFF_RAW + RAWS * RAW_BYTES + 1023) / 1024 * 1024;
  static constexpr int OFF_BAR = OFF_EPI + (FFN ? 0 : EW * EPI_RING * BOX_BYTES);  // (the FFN epilogues stage nothing)
  static constexpr int NUM_BARS = 2 * STAGES + 2 * SFS + 2 * RAWS + 2 * ACCB;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_TABLE = (OFF_MISC + 16 + 15) / 16 * 16;
  // grouped layouts: token-tile table; contiguous pairs: + the pair-unit table
  static constexpr int table_bytes(int form) {
    return form == kFormDense ? 0 : (form == kFormContig && PAIR ? 2 : 1) * kTableMax * 4;
  }
  static constexpr int smem_bytes(int form) { return OFF_TABLE + table_bytes(form) + 1024; }
  static_assert(EPI != 2 || smem_bytes(kFormKGrouped) <= 232448, "shared memory per CTA");

  static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "swizzle atoms");
  static_assert(OFF_SF % 128 == 0 && OFF_RAW % 128 == 0 && RAW_BYTES % 128 == 0,
                "scale groups and staged scales: 128-byte aligned");
  static_assert(EPI == 2 || smem_bytes(kFormContig) <= 232448, "shared memory per CTA");
};

// 16-byte chunk c (columns 8c .. 8c + 7) of row r of a 32-row x 64-byte box
// in the 64-byte swizzled layout of the tensor map: chunk bits 4-5 of the
// offset are XORed with bits 7-8, i.e. with (r / 2) % 4.
__device__ __forceinline__ int sw64_offset(int r, int c) { return r * 64 + ((c ^ ((r >> 1) & 3)) << 4); }

// UE8M0 byte of an fp32 power of two: its biased exponent.
__device__ __forceinline__ uint32_t ue8m0_byte(float s) { return (__float_as_uint(s) >> 23) & 0xFFu; }

// A scale this kernel cannot apply exactly: not +0 or a positive power of two
// (sign bit or mantissa bits set), or an infinity / NaN (exponent field 255).
__device__ __forceinline__ bool not_pow2_scale(float s) {
  const uint32_t u = __float_as_uint(s);
  return (u & 0x807FFFFFu) != 0u || (u >> 23) == 0xFFu;
}

// Tables of the grouped layouts, built by warp 0 before the main loops.
// Contiguous: table[mt] = expert of token tile mt (from its first row; -1 for
// padding tiles); with pairs also units[u] = first token tile of pair unit u
// and *num_units. Masked: table[e] = exclusive prefix over experts of the
// number of (token tile or tile pair, weight tile) work items.
template <class C, int FORM>
__device__ void mx_build_table(const GemmParams& p, int* table, int* num_units, int lane) {
  if constexpr (FORM == kFormContig) {
    for (int mt = lane; mt < p.num_mt; mt += 32) {
      int v = __ldg(p.m_indices + static_cast<int64_t>(mt) * C::BT);
      if (v >= p.G) {
        raise_status(p.status, 3 /* FG_DEVICE_BAD_M_INDEX */);
        v = -1;
      }
      table[mt] = v < 0 ? -1 : v;
    }
    if constexpr (C::PAIR) {
      __syncwarp();
      int* units = table + kTableMax;
      int count = 0;
      int run_start = 0;  // first tile of the run the previous chunk ended in
      int prev_e = -2;    // expert of the previous chunk's last tile
      for (int base = 0; base < p.num_mt; base += 32) {
        const int mt = base + lane;
        const int e = mt < p.num_mt ? table[mt] : -3;
        int e_before = __shfl_up_sync(0xffffffffu, e, 1);
        if (lane == 0) e_before = prev_e;
        // start of this tile's run: the last run start at or before it
        int rs = (mt < p.num_mt && e != e_before) ? mt : -1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, rs, o);
          if (lane >= o) rs = max(rs, v);
        }
        if (rs < 0) rs = run_start;
        // a unit starts at every other tile of a run of one expert
        const bool unit = mt < p.num_mt && e >= 0 && ((mt - rs) & 1) == 0;
        const unsigned bal = __ballot_sync(0xffffffffu, unit);
        if (unit) units[count + __popc(bal & ((1u << lane) - 1u))] = mt;
        count += __popc(bal);
        run_start = __shfl_sync(0xffffffffu, rs, 31);
        prev_e = __shfl_sync(0xffffffffu, e, 31);
      }
      if (lane == 0) *num_units = count;
    }
  } else if constexpr (FORM == kFormKGrouped) {
    // table[e] = first token block of expert e (exclusive prefix of ks / 128)
    const int per = (p.G + 31) / 32;
    const int e0 = lane * per;
    const int e1 = min(p.G, e0 + per);
    int local = 0;
    for (int e = e0; e < e1; ++e) {
      int k = __ldg(p.ks + e);
      if (k < 0 || (k & 127) != 0) {
        raise_status(p.status, 4 /* FG_DEVICE_BAD_K_GROUP */);
        k = k < 0 ? 0 : k & ~127;
      }
      table[e + 1] = k >> 7;
      local += k >> 7;
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
      table[e + 1] = min(run, p.KB);  // token blocks past T are dropped (status raised below)
    }
    if (lane == 31 && incl > p.KB) raise_status(p.status, 4 /* FG_DEVICE_BAD_K_GROUP */);
    if (lane == 0) table[0] = 0;
  } else if constexpr (FORM == kFormMasked) {
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
      int rows = (mm + C::BT - 1) / C::BT;  // token tiles
      if (C::PAIR) rows = (rows + 1) / 2;    // ... or tile pairs
      // (one-kernel FFN: the prefix counts token tiles or pairs; both GEMMs'
      // tiles are laid over them)
      const int cnt = C::FUSED ? rows : rows * p.num_nt;
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

// One-kernel FFN: token tiles (contiguous, single CTAs), pair units
// (contiguous pairs) or the masked prefix's tiles / pairs.
template <class C, int FORM>
__device__ __forceinline__ int mx_ffn_units(const GemmParams& p, const int* table, int num_units) {
  return FORM == kFormMasked ? table[p.G] : (C::PAIR ? num_units : p.num_mt);
}

template <class C, int FORM>
__device__ __forceinline__ int mx_total(const GemmParams& p, const int* table, int num_units) {
  if (C::FUSED) return mx_ffn_units<C, FORM>(p, table, num_units) * (p.num_nt + p.num_nt2);
  if (FORM == kFormMasked) return table[p.G];
  if (FORM == kFormKGrouped) return p.G * (C::PAIR ? (p.num_mt + 1) / 2 : p.num_mt) * p.num_nt;
  if (FORM == kFormContig && C::PAIR) return num_units * p.num_nt;
  return (C::PAIR ? (p.num_mt + 1) / 2 : p.num_mt) * p.num_nt;
}

// Work item t of this CTA (rank = its place in the pair; 0 without pairs).
// One-kernel FFN: items [0, t1) are the first GEMM's tiles, unit by unit (the
// num_nt tiles of a token tile or pair unit are consecutive), then the second
// GEMM's in the same order; `owned` says whether this CTA's token tile is the
// unit's own (a contiguous odd run's partner tile belongs to another expert
// or lies past the last tile; a masked pair's second tile may lie past M_max).
template <class C, int FORM>
__device__ __forceinline__ Tile mx_resolve(const GemmParams& p, const int* table, int t, int rank,
                                           int t1 = 0) {
  Tile w;
  w.valid = 1;
  w.kb0 = 0;
  w.nkb = p.KB;
  w.phase = 0;
  w.owned = 1;
  if constexpr (C::FUSED) {
    w.phase = t >= t1 ? 1 : 0;
    const int local = w.phase ? t - t1 : t;
    const int nts = w.phase ? p.num_nt2 : p.num_nt;
    const int u = local / nts;
    w.nt = local % nts;
    w.nkb = w.phase ? p.KB2 : p.KB;
    if (FORM == kFormMasked) {
      int lo = 0, hi = p.G;  // table[lo] <= u < table[hi]
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (table[mid] <= u) lo = mid; else hi = mid;
      }
      const int li = u - table[lo];
      w.e = lo;
      w.mt = C::PAIR ? 2 * li + rank : li;
      w.owned = w.mt < p.num_mt;
    } else if (C::PAIR) {
      const int mt0 = table[kTableMax + u];
      w.e = table[mt0];
      w.mt = mt0 + rank;
      w.owned = w.mt < p.num_mt && table[w.mt] == w.e;
    } else {
      w.mt = u;
      w.e = table[u];
      w.valid = w.e >= 0;
      w.owned = w.valid;
    }
    return w;
  }
  if (FORM == kFormKGrouped) {
    const int per = (C::PAIR ? (p.num_mt + 1) / 2 : p.num_mt) * p.num_nt;
    w.e = t / per;
    const int local = t - w.e * per;
    w.mt = C::PAIR ? 2 * (local / p.num_nt) + rank : local / p.num_nt;
    w.nt = local % p.num_nt;
    w.kb0 = table[w.e];
    w.nkb = table[w.e + 1] - table[w.e];
  } else if (FORM == kFormMasked) {
    int lo = 0, hi = p.G;  // table[lo] <= t < table[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (table[mid] <= t) lo = mid; else hi = mid;
    }
    const int local = t - table[lo];
    w.e = lo;
    w.mt = C::PAIR ? 2 * (local / p.num_nt) + rank : local / p.num_nt;
    w.nt = local % p.num_nt;
  } else if (FORM == kFormContig && C::PAIR) {
    const int mt0 = table[kTableMax + t / p.num_nt];
    w.e = table[mt0];
    w.mt = mt0 + rank;
    w.nt = t % p.num_nt;
  } else {
    w.mt = C::PAIR ? 2 * (t / p.num_nt) + rank : t / p.num_nt;
    w.nt = t % p.num_nt;
    if (FORM == kFormContig) {
      w.e = table[w.mt];
      w.valid = w.e >= 0;
    } else {
      w.e = 0;
    }
  }
  return w;
}

// Accumulator of a CTA's next tile: the tiles take the accumulators in turn
// (ACC of them); the one-kernel FFN's first-GEMM tiles always use the
// 256-column accumulator 0, its second-GEMM tiles alternate between two
// 224-column ones starting with 0 (so the first of them waits for the last
// first-GEMM tile's epilogue, whose columns the second one overlaps).
// uses(b) counts the tiles accumulator b has held (its barriers' parity);
// k1 counts the second-GEMM tiles seen.
template <class C>
struct AccTurn {
  static_assert(C::ACCB == 1 || C::ACCB == 2, "one or two accumulators");
  uint32_t u0 = 0, u1 = 0;  // tiles accumulator 0 / 1 has held (its barriers' parity)
  uint32_t tiles = 0, k1 = 0;
  __device__ __forceinline__ int next(const Tile& w) const {
    if constexpr (C::FUSED) return w.phase ? static_cast<int>(k1 & 1u) : 0;
    return static_cast<int>(tiles % C::ACC);
  }
  __device__ __forceinline__ uint32_t uses(int b) const { return b ? u1 : u0; }
  __device__ __forceinline__ void done(const Tile& w, int b) {
    if (b) ++u1; else ++u0;
    ++tiles;
    if (C::FUSED && w.phase) ++k1;
  }
  // first tensor-memory column of accumulator b for tile w
  __device__ __forceinline__ static uint32_t column(const Tile& w, int b) {
    return static_cast<uint32_t>(C::FUSED ? (w.phase ? b * C::BW2 : 0) : b * C::BW);
  }
};

// Position in a ring of N slots, advanced one use at a time: slot index and
// the parity of the slot's current phase.
template <int N>
struct Ring {
  uint32_t slot = 0, phase = 0;
  __device__ __forceinline__ void next() {
    if (++slot == N) {
      slot = 0;
      phase ^= 1u;
    }
  }
};

template <class C, int FORM>
__global__ void __launch_bounds__(C::NUM_THREADS, 1)
    fp8_gemm_mx_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                       const __grid_constant__ CUtensorMap tmD, const __grid_constant__ CUtensorMap tmA2,
                       const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ CUtensorMap tmSA2,
                       const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem + C::OFF_A;
  uint8_t* sB = smem + C::OFF_B;
  uint8_t* sSF = smem + C::OFF_SF;
  uint8_t* sRAW = smem + C::OFF_RAW;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + C::STAGES;
  uint64_t* sf_full = empty + C::STAGES;    // a scale slot's groups are written (both CTAs)
  uint64_t* sf_empty = sf_full + C::SFS;    // ... and the quad's MMAs have completed
  uint64_t* sa_full = sf_empty + C::SFS;    // a quad's fp32 scales have landed
  uint64_t* sa_empty = sa_full + C::RAWS;   // ... and the converter has read them
  uint64_t* tfull = sa_empty + C::RAWS;     // an accumulator holds a finished tile
  uint64_t* tempty = tfull + C::ACCB;       // ... and has been read by the epilogue
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  int* table = reinterpret_cast<int*>(smem + C::OFF_TABLE);
  int* num_units = reinterpret_cast<int*>(smem + C::OFF_MISC + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = C::PAIR ? static_cast<int>(cluster_ctarank()) : 0;
  const int t_first = C::PAIR ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
  const int t_step = C::PAIR ? static_cast<int>(num_clusters_x()) : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 2);      // weight- and token-tile lanes' expect_tx (the leader's, for a pair)
      mbar_init(&empty[s], 1);     // the MMA commit
    }
    for (int q = 0; q < C::SFS; ++q) {
      mbar_init(&sf_full[q], C::CLUSTER);  // the converter warp of each CTA
      mbar_init(&sf_empty[q], 1);          // the MMA commit after the quad
    }
    for (int r = 0; r < C::RAWS; ++r) {
      // scale lane: expect_tx (TMA), plus the cp.async arrival (weight-block scales)
      mbar_init(&sa_full[r], C::EPI == 2 ? 1 : 2);
      mbar_init(&sa_empty[r], 1);  // the converter
    }
    for (int b = 0; b < C::ACCB; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], C::CLUSTER * C::EW);  // one arrival per epilogue warp (of both CTAs)
    }
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmSA);
    if (C::EPI == 2) tma_prefetch_desc(&tmSB);
    if (!C::FFN) tma_prefetch_desc(&tmD);
    if (C::FUSED) {
      // the second GEMM's operands: the quantized activations, W2 and sfh
      tma_prefetch_desc(&tmA2);
      tma_prefetch_desc(&tmB2);
      tma_prefetch_desc(&tmSA2);
    }
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
  if constexpr (C::PAIR) cluster_arrive_relaxed();
  // Everything above may overlap the previous kernel; memory comes after this.
  grid_dependency_wait();
  if (warp == 0) mx_build_table<C, FORM>(p, table, num_units, lane);
  tc_fence_before();
  __syncthreads();
  if constexpr (C::PAIR) {
    cluster_wait();
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
  const uint32_t tmem_sf = tmem_base + static_cast<uint32_t>(C::SF_BASE);
  const WaitCtl ctl{abort_flag, p.status, p.timeout_ns};
  const int total = mx_total<C, FORM>(p, table, *num_units);
  // one-kernel FFN: the first GEMM's items come first
  const int t1 = C::FUSED ? mx_ffn_units<C, FORM>(p, table, *num_units) * p.num_nt : 0;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane < 2) {
      Ring<C::STAGES> st;
      uint32_t fills = 0;
      for (int t = t_first; t < total; t += t_step) {
        const Tile w = mx_resolve<C, FORM>(p, table, t, rank, t1);
        if (!w.valid) continue;
        // fused FFN: gate block nt*128.. and up block I + nt*128.. of the
        // expert's 2I rows (a pair's CTAs load one block each)
        // (K-grouped: B is one matrix whose K range the experts share)
        // (one-kernel FFN, second GEMM: BW consecutive rows of the expert's
        // W2 and the tile's rows of the quantized activations)
        const bool ffn_tile = C::EPI == 1 || (C::FUSED && w.phase == 0);
        const bool second = C::FUSED && w.phase == 1;
        const int b_base = FORM == kFormKGrouped ? 0 : w.e * (second ? p.N2 : p.N);
        const int row = lane == 0 ? (ffn_tile ? b_base + (C::PAIR ? rank : 0) * p.I + w.nt * 128
                                   : second ? b_base + w.nt * C::BW2 + rank * C::B_ROWS2
                                            : b_base + w.nt * C::BW + rank * C::B_ROWS)
                                  : (FORM == kFormMasked ? w.e * p.M : 0) + w.mt * C::BT;
        const CUtensorMap* map = lane == 0 ? (second ? &tmB2 : &tmB) : (second ? &tmA2 : &tmA);
        // K block j of a stage sits at j * stride; `bytes` of it are loaded
        // (the second GEMM's B_ROWS2-row weight tiles leave the rest unused)
        const uint32_t stride = lane == 0 ? C::B_BYTES : C::A_BYTES;
        const uint32_t bytes = lane == 0 ? (second ? C::B_ROWS2 * 128 : C::B_BYTES) : C::A_BYTES;
        const int loads = lane == 0 && !second ? C::B_LOADS : 1;  // tensor loads per K block
        const int load_step = ffn_tile ? p.I : C::B_BOX;         // rows between them
        if (second && lane == 1 && w.owned) {
          // the tile's quantized activations are complete (every first-GEMM
          // tile of this token tile has published its rows)
          const int ri = (FORM == kFormMasked ? w.e * p.num_mt : 0) + w.mt;
          if (!wait_counter(p.ready + ri, p.ready_target, abort_flag, p.status, p.timeout_ns))
            goto producer_done;
          fence_proxy_async_global();  // the tensor loads below read them
        }
        for (int kb0 = 0; kb0 < w.nkb; kb0 += C::KPS, st.next(), ++fills) {
          if (!mbar_wait(&empty[st.slot], st.phase ^ 1u, ctl)) goto producer_done;
          const int nk = min(C::KPS, w.nkb - kb0);
          const int kx = (w.kb0 + kb0) * 128;  // K coordinate of the stage's first block
          uint8_t* dst = lane == 0 ? sB + st.slot * C::STAGE_B : sA + st.slot * C::STAGE_A;
          if constexpr (C::PAIR) {
            // both CTAs' operand bytes complete on the leader's barrier
            if (rank == 0) mbar_arrive_expect_tx(&full[st.slot], 2 * nk * bytes);
            const uint32_t bar = mapa_shared(smem_u32(&full[st.slot]), 0);
            for (int j = 0; j < nk; ++j)
              for (int h = 0; h < loads; ++h)
                tma_load_2d_pair(dst + j * stride + h * C::B_BOX * 128, map, bar, kx + j * 128,
                                 row + h * load_step);
          } else {
            mbar_arrive_expect_tx(&full[st.slot], nk * bytes);
            for (int j = 0; j < nk; ++j)
              for (int h = 0; h < loads; ++h)
                tma_load_2d(dst + j * stride + h * C::B_BOX * 128, map, &full[st.slot], kx + j * 128,
                            row + h * load_step);
          }
        }
      }
    producer_done:
      // the last fill of every stage has landed and been consumed before the
      // CTA releases its shared memory
      if (lane == 0) {
        for (uint32_t s = 0; s < C::STAGES && s < fills; ++s) {
          const uint32_t last = (fills - 1 - s) / C::STAGES * C::STAGES + s;
          // (a pair's operand bytes complete on the leader's barrier)
          if (!C::PAIR || rank == 0) drain_wait(&full[last % C::STAGES], (last / C::STAGES) & 1u, kDrainLimitNs);
          drain_wait(&empty[last % C::STAGES], (last / C::STAGES) & 1u, kDrainLimitNs);
        }
      }
    } else if (lane == 2) {
      Ring<C::RAWS> rr;
      uint32_t fills = 0;
      for (int t = t_first; t < total; t += t_step) {
        const Tile w = mx_resolve<C, FORM>(p, table, t, rank, t1);
        if (!w.valid) continue;
        // weight blocks the tile's rows touch (clamped: rows past N are never stored)
        const bool ffn_tile = C::EPI == 1 || (C::FUSED && w.phase == 0);
        const bool second = C::FUSED && w.phase == 1;
        const int NB = second ? p.NB2 : p.NB;
        const int KB = second ? p.KB2 : p.KB;
        const int nb0 = (w.nt * (second ? C::BW2 : C::BW)) >> 7;
        const float* sfb_e = (second ? p.sfb2 : p.sfb) + static_cast<int64_t>(w.e) * NB * KB;
        if (second && w.owned) {
          // the tile's token scales are written by the first GEMM's epilogue
          const int ri = (FORM == kFormMasked ? w.e * p.num_mt : 0) + w.mt;
          if (!wait_counter(p.ready + ri, p.ready_target, abort_flag, p.status, p.timeout_ns))
            goto scales_done;
          fence_proxy_async_global();
        }
        const int KQ = (w.nkb + 3) >> 2;  // quads of the tile
        for (int qi = 0; qi < KQ; ++qi, rr.next(), ++fills) {
          if (!mbar_wait(&sa_empty[rr.slot], rr.phase ^ 1u, ctl)) goto scales_done;
          uint8_t* raw = sRAW + rr.slot * C::RAW_BYTES;
          // 4 K blocks of token scales; rows past M read as zero, K blocks past
          // the tile's last one are never used
          const int ky = (FORM == kFormMasked ? w.e * KB : 0) + w.kb0 + 4 * qi;
          if constexpr (C::EPI == 2) {
            // per-row weight scales: BW rows x 4 K blocks beside them
            mbar_arrive_expect_tx(&sa_full[rr.slot], C::RAW_A + C::RAW_B);
            tma_load_2d(raw, &tmSA, &sa_full[rr.slot], w.mt * C::BT, ky);
            tma_load_2d(raw + C::RAW_A, &tmSB, &sa_full[rr.slot], w.nt * C::BW, ky);
            continue;
          }
          mbar_arrive_expect_tx(&sa_full[rr.slot], C::RAW_A);
          tma_load_2d(raw, second ? &tmSA2 : &tmSA, &sa_full[rr.slot], w.mt * C::BT, ky);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int kb = w.kb0 + min(4 * qi + k, w.nkb - 1);
#pragma unroll
            for (int j = 0; j < C::NBT; ++j) {
              // fused FFN: the gate block nt and the up block I/128 + nt (a
              // third staged block, where the config has one, repeats it)
              const int nb = ffn_tile ? (j == 0 ? w.nt : (p.I >> 7) + w.nt) : min(nb0 + j, NB - 1);
              cp_async_4(raw + C::RAW_A + 4 * (k * C::NBT + j), sfb_e + static_cast<int64_t>(nb) * KB + kb);
            }
          }
          cp_async_mbar_arrive(&sa_full[rr.slot]);
        }
      }
    scales_done:
      for (uint32_t r = 0; r < C::RAWS && r < fills; ++r) {
        const uint32_t last = (fills - 1 - r) / C::RAWS * C::RAWS + r;
        drain_wait(&sa_full[last % C::RAWS], (last / C::RAWS) & 1u, kDrainLimitNs);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (converged, so that descriptors and
    // addresses stay warp-uniform); one elected lane issues the tcgen05
    // instructions, the same lane every time (copies and the MMAs that read
    // them must come from one thread).
    if (rank == 0) {  // a pair's MMAs are issued by its leader
      constexpr uint32_t idesc1 = mma_idesc_e4m3_bs(C::MMA_M, C::BW);
      constexpr uint32_t idesc2 = mma_idesc_e4m3_bs(C::MMA_M, C::BW2);  // (one-kernel FFN, second GEMM)
      Ring<C::STAGES> st;
      Ring<C::SFS> sq;
      AccTurn<C> acc;
      int last_b = 0;
      bool ready = false;  // the current stage's "full" phase was seen complete by a peek
      for (int t = t_first; t < total; t += t_step) {
        const Tile w = mx_resolve<C, FORM>(p, table, t, rank, t1);
        if (!w.valid || w.nkb == 0) continue;  // (an expert without tokens: no MMA)
        const int b = acc.next(w);
        if (!warp_wait(&tempty[b], (acc.uses(b) & 1u) ^ 1u, ctl, lane)) goto mma_done;
        tc_fence_after();
        const uint32_t d = tmem_base + AccTurn<C>::column(w, b);
        const uint32_t idesc = C::FUSED && w.phase ? idesc2 : idesc1;
        for (int kb0 = 0; kb0 < w.nkb; kb0 += C::KPS, st.next()) {
          if (!ready && !warp_wait(&full[st.slot], st.phase, ctl, lane)) goto mma_done;
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + st.slot * C::STAGE_A);
          const uint32_t b_base = smem_u32(sB + st.slot * C::STAGE_B);
#pragma unroll
          for (int j = 0; j < C::KPS; ++j) {
            const int kb = kb0 + j;
            if (kb >= w.nkb) break;
            const uint32_t k4 = static_cast<uint32_t>(kb & 3);
            const uint32_t sf = tmem_sf + sq.slot * C::SF_COLS;
            if (k4 == 0) {
              // a new quad: its scale groups (both CTAs') into tensor memory
              if (!warp_wait(&sf_full[sq.slot], sq.phase, ctl, lane)) goto mma_done;
              tc_fence_after();
              const uint32_t src = smem_u32(sSF + sq.slot * C::SF_BYTES);
              if (elect_one()) {
#pragma unroll
                for (int g = 0; g <= C::SFB_GROUPS; ++g) {
                  if constexpr (C::PAIR) tmem_cp_sf_group_pair(sf + 4 * g, src + 512 * g);
                  else tmem_cp_sf_group(sf + 4 * g, src + 512 * g);
                }
              }
            }
            // byte k4 of each scale word: this K block's scales
            const uint32_t sfa = sf | (k4 << 30);
            const uint32_t sfb = (sf + 4) | (k4 << 30);
            const uint32_t id = idesc | (k4 << 4) | (k4 << 29);
            const uint64_t adesc = smem_desc_sw128(a_base + j * C::A_BYTES);
            const uint64_t bdesc = smem_desc_sw128(b_base + j * C::B_BYTES);
            const bool last_of_quad = k4 == 3 || kb == w.nkb - 1;
            if (elect_one()) {
#pragma unroll
              for (int k = 0; k < 4; ++k) {  // 32 bytes (= 32 e4m3 along K) per MMA
                if constexpr (C::PAIR)
                  mma_f8_bs_pair(d, adesc + 2 * k, bdesc + 2 * k, id, sfa, sfb, (kb | k) != 0 ? 1u : 0u);
                else
                  mma_f8_bs(d, adesc + 2 * k, bdesc + 2 * k, id, sfa, sfb, (kb | k) != 0 ? 1u : 0u);
              }
              if (last_of_quad) {
                // the quad's scale slot is free once these MMAs complete
                if constexpr (C::PAIR) mma_commit_pair(&sf_empty[sq.slot]);
                else mma_commit(&sf_empty[sq.slot]);
              }
            }
            if (last_of_quad) sq.next();
          }
          // peek at the next stage while this stage's MMAs execute
          {
            Ring<C::STAGES> nx = st;
            nx.next();
            ready = __all_sync(0xffffffffu, mbar_test_wait(&full[nx.slot], nx.phase));
          }
          if (elect_one()) {
            if constexpr (C::PAIR) mma_commit_pair(&empty[st.slot]);  // both CTAs' stage
            else mma_commit(&empty[st.slot]);
          }
        }
        if (elect_one()) {
          if constexpr (C::PAIR) mma_commit_pair(&tfull[b]);
          else mma_commit(&tfull[b]);
        }
        acc.done(w, b);
        last_b = b;
      }
    mma_done:
      if (acc.tiles > 0 && lane == 0)
        drain_wait(&tfull[last_b], (acc.uses(last_b) - 1) & 1u, kDrainLimitNs);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ scale converter
    Ring<C::RAWS> rr;
    Ring<C::SFS> sq;
    for (int t = t_first; t < total; t += t_step) {
      const Tile w = mx_resolve<C, FORM>(p, table, t, rank, t1);
      if (!w.valid) continue;
      // staged weight-block index of this lane's weight rows lane + 32 r1 + 128 g
      // (a first-GEMM FFN tile: group 0 = the gate block, 1 = the up block)
      const bool ffn_tile = C::EPI == 1 || (C::FUSED && w.phase == 0);
      const int n0 = w.nt * (C::FUSED && w.phase ? C::BW2 : C::BW);
      int jb[C::SFB_GROUPS][4];
#pragma unroll
      for (int g = 0; g < C::SFB_GROUPS; ++g)
#pragma unroll
        for (int r1 = 0; r1 < 4; ++r1)
          jb[g][r1] = ffn_tile ? g : ((n0 + 128 * g + 32 * r1 + lane) >> 7) - (n0 >> 7);
      // rows of this lane (lane + 32 r1) whose outputs are stored: only their
      // token scales must be powers of two (rows past M arrive as zeros;
      // masked rows past masked_m and contiguous rows of another expert or
      // padding hold whatever the caller left there)
      uint32_t rows_ok = 0xFu;
      if constexpr (FORM == kFormMasked) {
        int mv = __ldg(p.masked_m + w.e);
        mv = mv < 0 ? 0 : (mv > p.M ? p.M : mv);
#pragma unroll
        for (int r1 = 0; r1 < 4; ++r1)
          if (w.mt * C::BT + 32 * r1 + lane >= mv) rows_ok &= ~(1u << r1);
      } else if constexpr (FORM == kFormContig) {
#pragma unroll
        for (int r1 = 0; r1 < 4; ++r1) {
          const int m = w.mt * C::BT + 32 * r1 + lane;
          if (m >= p.M || __ldg(p.m_indices + m) != w.e) rows_ok &= ~(1u << r1);
        }
      }
      bool bad_scale = false;
      const int KQ = (w.nkb + 3) >> 2;  // quads of the tile
      for (int qi = 0; qi < KQ; ++qi, rr.next(), sq.next()) {
        // the quad's scales have landed, and the slot's previous quad has
        // been copied out and its MMAs have completed
        if (!warp_wait(&sa_full[rr.slot], rr.phase, ctl, lane)) goto convert_done;
        if (!warp_wait(&sf_empty[sq.slot], sq.phase ^ 1u, ctl, lane)) goto convert_done;
        const float* raw = reinterpret_cast<const float*>(sRAW + rr.slot * C::RAW_BYTES);
        const int nk = min(4, w.nkb - 4 * qi);  // K blocks of this quad
        uint32_t wa[4] = {0, 0, 0, 0};
        uint32_t wb[C::SFB_GROUPS][4];
#pragma unroll
        for (int g = 0; g < C::SFB_GROUPS; ++g)
#pragma unroll
          for (int r1 = 0; r1 < 4; ++r1) wb[g][r1] = 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (k < nk) {
#pragma unroll
            for (int r1 = 0; r1 < 4; ++r1) {
              const float sa = raw[k * 128 + 32 * r1 + lane];
              bad_scale |= ((rows_ok >> r1) & 1u) && not_pow2_scale(sa);
              wa[r1] |= ue8m0_byte(sa) << (8 * k);
            }
#pragma unroll
            for (int g = 0; g < C::SFB_GROUPS; ++g)
#pragma unroll
              for (int r1 = 0; r1 < 4; ++r1) {
                if constexpr (C::EPI == 2) {
                  // per-row weight scale of tile row 128 g + 32 r1 + lane
                  const int n = 128 * g + 32 * r1 + lane;
                  const float sb = n < C::BW ? raw[C::RAW_A / 4 + k * C::BW + n] : 1.0f;
                  bad_scale |= not_pow2_scale(sb);
                  wb[g][r1] |= (n < C::BW ? ue8m0_byte(sb) : 127u) << (8 * k);
                } else {
                  // (blocks past the weight's last one arrive as zeros)
                  const float sb = raw[C::RAW_A / 4 + k * C::NBT + jb[g][r1]];
                  bad_scale |= not_pow2_scale(sb);
                  wb[g][r1] |= ue8m0_byte(sb) << (8 * k);
                }
              }
          }
        }
        uint8_t* grp = sSF + sq.slot * C::SF_BYTES + lane * 16;
        *reinterpret_cast<uint4*>(grp) = make_uint4(wa[0], wa[1], wa[2], wa[3]);
#pragma unroll
        for (int g = 0; g < C::SFB_GROUPS; ++g)
          *reinterpret_cast<uint4*>(grp + 512 * (1 + g)) = make_uint4(wb[g][0], wb[g][1], wb[g][2], wb[g][3]);
        // visible to this CTA's async proxy (which executes tcgen05.cp for
        // this CTA's shared memory, also when the leader issues it) before
        // the arrival leaves this thread
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sa_empty[rr.slot]);
          // (a remote arrival with cluster-scope release stalls the issuing
          // thread for about a microsecond; the leader issues the copy only
          // after observing this arrival, by which time the writes above are
          // visible to the async proxy)
          if (C::PAIR && rank != 0)
            mbar_arrive_remote(mapa_shared(smem_u32(&sf_full[sq.slot]), 0));
          else
            mbar_arrive(&sf_full[sq.slot]);
        }
      }
      // a scale the block-scaled MMA would round: the call's result is wrong
      if (__any_sync(0xffffffffu, bad_scale) && lane == 0)
        raise_status(p.status, 5 /* FG_DEVICE_BAD_SCALE */);
    }
  convert_done:;
  } else if (C::FFN && warp >= C::EPI_BASE) {
    // ------------------------------------------------------------ fused FFN epilogue
    const int quad = warp & 3;          // TMEM lanes this warp may access (one warp per quadrant)
    const int row = quad * 32 + lane;   // token row of this CTA's tile
    const uint32_t t_lane = static_cast<uint32_t>(quad * 32) << 16;
    const int IB = p.I >> 7;
    AccTurn<C> acc;
    for (int t = t_first; t < total; t += t_step) {
      const Tile w = mx_resolve<C, FORM>(p, table, t, rank, t1);
      if (!w.valid) continue;
      int m_valid = p.M;
      if (FORM == kFormMasked) {
        m_valid = __ldg(p.masked_m + w.e);
        m_valid = m_valid < 0 ? 0 : (m_valid > p.M ? p.M : m_valid);
      }
      const int m = w.mt * C::BT + row;
      bool ok = m < m_valid;
      if (FORM == kFormContig) ok = ok && __ldg(p.m_indices + m) == w.e;
      const int64_t grow = (FORM == kFormMasked ? static_cast<int64_t>(w.e) * p.M : 0) + m;
      const int b = acc.next(w);
      if (!warp_wait(&tfull[b], acc.uses(b) & 1u, ctl, lane)) goto ffn_done;
      tc_fence_after();
      if (C::FUSED && w.phase == 1) {
        // one-kernel FFN, second GEMM: the row's BW2 accumulator columns as
        // packed bf16, the accumulator released (the next tile's MMAs run in
        // the other one meanwhile), then Y written directly
        constexpr int YW = C::BW2 / 2;  // packed pairs
        uint32_t yp[YW];
        const uint32_t a0 = tmem_base + t_lane + AccTurn<C>::column(w, b);
#pragma unroll
        for (int c = 0; c < C::BW2 / 32; ++c) {
          uint32_t r0[32];
          tmem_ld32_issue(a0 + static_cast<uint32_t>(32 * c), r0);
          tmem_wait_ld32(r0);
#pragma unroll
          for (int j = 0; j < 16; ++j)
            yp[16 * c + j] = pack_bf16x2(__uint_as_float(r0[2 * j]), __uint_as_float(r0[2 * j + 1]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (C::PAIR && rank != 0) mbar_arrive_remote(mapa_shared(smem_u32(&tempty[b]), 0));
          else mbar_arrive(&tempty[b]);
        }
        if (ok) {
          const int x0 = w.nt * C::BW2;  // columns past H (a last, partial tile) are not stored
          uint16_t* ydst = p.D + grow * p.N2 + x0;
#pragma unroll
          for (int j = 0; j < YW; j += 4)
            if (x0 + 2 * j < p.N2)
              *reinterpret_cast<uint4*>(ydst + 2 * j) = make_uint4(yp[j], yp[j + 1], yp[j + 2], yp[j + 3]);
        }
        acc.done(w, b);
        continue;
      }
      // gate and up values as packed bf16 pairs (the activation takes them in
      // bf16): all 256 columns are read first, so that the accumulator goes
      // back to the MMA before the activation arithmetic
      uint32_t gp[64], upk[64];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t rg[32], ru[32];
        tmem_ld32_issue(tmem_base + t_lane + static_cast<uint32_t>(32 * c), rg);
        tmem_ld32_issue(tmem_base + t_lane + static_cast<uint32_t>(128 + 32 * c), ru);
        tmem_wait_ld64(rg, ru);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          gp[16 * c + j] = pack_bf16x2(__uint_as_float(rg[2 * j]), __uint_as_float(rg[2 * j + 1]));
          upk[16 * c + j] = pack_bf16x2(__uint_as_float(ru[2 * j]), __uint_as_float(ru[2 * j + 1]));
        }
      }
      // the accumulator is in registers: the next tile's MMAs may start
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (C::PAIR && rank != 0) mbar_arrive_remote(mapa_shared(smem_u32(&tempty[b]), 0));
        else mbar_arrive(&tempty[b]);
      }
      if (p.gu != nullptr && ok) {
        // bf16 gate at columns nt*128.., up at I + nt*128..
        uint16_t* gdst = p.gu + grow * (2 * p.I) + w.nt * 128;
#pragma unroll
        for (int j = 0; j < 64; j += 4) {
          *reinterpret_cast<uint4*>(gdst + 2 * j) = make_uint4(gp[j], gp[j + 1], gp[j + 2], gp[j + 3]);
          *reinterpret_cast<uint4*>(gdst + p.I + 2 * j) = make_uint4(upk[j], upk[j + 1], upk[j + 2], upk[j + 3]);
        }
      }
      if (ok) {
        // h = bf16(silu(gate) * up), kept as packed bf16 pairs, and its amax;
        // only for rows that are stored (padding rows are zeros, on which the
        // IEEE division of silu runs its slow path: a warp of them took twice
        // as long as a warp of tokens and held up the next tile)
        uint32_t hp[64];
        float amax = 0.0f;
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const float h0 = round_bf16(__fmul_rn(silu_fixed(bf16_lo(gp[j])), bf16_lo(upk[j])));
          const float h1 = round_bf16(__fmul_rn(silu_fixed(bf16_hi(gp[j])), bf16_hi(upk[j])));
          amax = fmaxf(amax, fmaxf(fabsf(h0), fabsf(h1)));
          hp[j] = pack_bf16x2(h0, h1);
        }
        // the per-token power-of-two quantization of per_token_cast_to_fp8_ue8m0
        float scale, inv;
        group_scale<true>(fmaxf(amax, kAmaxFloor), scale, inv);
        uint8_t* qdst = p.hq + grow * p.I + w.nt * 128;
#pragma unroll
        for (int j = 0; j < 64; j += 8) {
          uint32_t v[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            v[i] = static_cast<uint32_t>(cvt_e4m3x2(__fmul_rn(bf16_lo(hp[j + 2 * i]), inv),
                                                    __fmul_rn(bf16_hi(hp[j + 2 * i]), inv))) |
                   (static_cast<uint32_t>(cvt_e4m3x2(__fmul_rn(bf16_lo(hp[j + 2 * i + 1]), inv),
                                                     __fmul_rn(bf16_hi(hp[j + 2 * i + 1]), inv))) << 16);
          *reinterpret_cast<uint4*>(qdst + 2 * j) = make_uint4(v[0], v[1], v[2], v[3]);
        }
        p.sfh[static_cast<int64_t>((FORM == kFormMasked ? w.e * IB : 0) + w.nt) * p.sfh_stride + m] = scale;
      }
      if constexpr (C::FUSED) {
        if (w.owned) {
          // publish this warp's rows of the token tile to the second GEMM's
          // tensor loads (other CTAs): the lanes' stores, ordered before the
          // async proxy's later reads, then, after the warp barrier (which
          // orders every lane's stores before lane 0's next operations), one
          // count per warp with release semantics at GPU scope; the reader
          // acquires the count and fences its own proxy before loading.
          fence_proxy_async_global();
          __syncwarp();
          if (lane == 0)
            red_release_gpu_add(p.ready + (FORM == kFormMasked ? w.e * p.num_mt : 0) + w.mt, 1);
        }
      }
      acc.done(w, b);
    }
  ffn_done:;
  } else if (warp >= C::EPI_BASE) {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - C::EPI_BASE;
    const int quad = warp & 3;          // TMEM lanes this warp may access
    const int c0 = (ew >> 2) * C::ECOLS;
    const int row = quad * 32 + lane;   // token row of this CTA's tile
    const uint32_t t_lane = static_cast<uint32_t>(quad * 32) << 16;
    uint8_t* ring = smem + C::OFF_EPI + ew * C::EPI_RING * C::BOX_BYTES;
    uint32_t tc = 0, boxes = 0;
    for (int t = t_first; t < total; t += t_step) {
      const Tile w = mx_resolve<C, FORM>(p, table, t, rank, t1);
      if (!w.valid) continue;
      int m_valid = p.M;
      if (FORM == kFormMasked) {
        m_valid = __ldg(p.masked_m + w.e);
        m_valid = m_valid < 0 ? 0 : (m_valid > p.M ? p.M : m_valid);
      }
      const int m = w.mt * C::BT + row;
      int row_mi = 0;
      // contiguous: a row is stored if it belongs to the tile's expert (rows of
      // padding, and rows of a pair unit's partner tile that belong to another
      // expert, are not)
      if (FORM == kFormContig) row_mi = (m < p.M && __ldg(p.m_indices + m) == w.e) ? 0 : -1;
      const bool ok = m < m_valid && (FORM != kFormContig || row_mi >= 0);
      // a warp whose 32 rows are all stored writes through tensor stores
      const bool staged = __all_sync(0xffffffffu, ok);
      const int y = (FORM == kFormMasked || FORM == kFormKGrouped ? w.e * p.M : 0) + w.mt * C::BT + quad * 32;
      const bool zero = w.nkb == 0;  // K-grouped expert without tokens: zeros, no accumulator
      const int b = tc % C::ACC;
      if (!zero) {
        if (!warp_wait(&tfull[b], (tc / C::ACC) & 1u, ctl, lane)) goto epi_done;
        tc_fence_after();
      }
#pragma unroll 1
      for (int ch = 0; ch < C::ECOLS / 32; ++ch) {
        uint32_t r[32];
        if (zero) {
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = 0u;
        } else {
          tmem_ld32_issue(tmem_base + t_lane + static_cast<uint32_t>(b * C::BW + c0 + ch * 32), r);
          tmem_wait_ld32(r);
          if (ch == C::ECOLS / 32 - 1) {
            // the accumulator is in registers: the next tile's MMAs may start
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              if (C::PAIR && rank != 0)  // the leader's MMA waits for both CTAs
                mbar_arrive_remote(mapa_shared(smem_u32(&tempty[b]), 0));
              else
                mbar_arrive(&tempty[b]);
            }
          }
        }
        const int x = w.nt * C::BW + c0 + ch * 32;
        if (staged) {
          uint8_t* img = ring + (boxes % C::EPI_RING) * C::BOX_BYTES;
          // the tensor store that last used this buffer has read it
          if (boxes >= C::EPI_RING && lane == 0) bulk_wait_group_read<C::EPI_RING - 1>();
          __syncwarp();
          if constexpr (C::EPI == 2) {
            // fp32: row `lane` of the box is 128 bytes; 16-byte chunk c at
            // position c ^ (lane % 8) (the tensor map's 128-byte swizzle)
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(img + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                  make_uint4(r[4 * c], r[4 * c + 1], r[4 * c + 2], r[4 * c + 3]);
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c)
              *reinterpret_cast<uint4*>(img + sw64_offset(lane, c)) = make_uint4(
                  pack_bf16x2(__uint_as_float(r[8 * c + 0]), __uint_as_float(r[8 * c + 1])),
                  pack_bf16x2(__uint_as_float(r[8 * c + 2]), __uint_as_float(r[8 * c + 3])),
                  pack_bf16x2(__uint_as_float(r[8 * c + 4]), __uint_as_float(r[8 * c + 5])),
                  pack_bf16x2(__uint_as_float(r[8 * c + 6]), __uint_as_float(r[8 * c + 7])));
          }
          fence_proxy_async_shared();
          __syncwarp();
          if (lane == 0) {
            if (x < p.N) tma_store_2d(&tmD, img, x, y);  // columns past N are clipped
            bulk_commit_group();  // (possibly empty: keeps one group per buffer use)
          }
          ++boxes;
        } else if constexpr (C::EPI == 2) {
          if (ok) {
            float* dst = p.d32 + (static_cast<int64_t>(w.e) * p.M + m) * p.N;
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              if (x + j < p.N) *reinterpret_cast<uint4*>(dst + x + j) = make_uint4(r[j], r[j + 1], r[j + 2], r[j + 3]);
          }
        } else {
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
          store_tile_part<C, FORM, 32>(p, w, row, c0 + ch * 32, v, m_valid, row_mi);
        }
      }
      if (!zero) ++tc;
    }
  epi_done:
    // this warp's tensor stores have finished reading shared memory
    if (lane == 0) bulk_wait_group_read<0>();
  }

  // ---------------------------------------------------------------- teardown
  __syncwarp();
  tc_fence_before();
  if constexpr (C::PAIR) {
    // each CTA arrives only after the MMAs writing its tensor memory and
    // reading its shared memory have completed (drained above)
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
