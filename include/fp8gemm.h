/*
 * fp8gemm.h - C ABI of the B200 (sm_100a) FP8 block-scaled GEMM library.
 *
 * The library computes D[bf16] = (A * sa)(B * sb)^T where A and B hold FP8
 * e4m3 codes, A carries one fp32 scale per token per 128-channel slice and B
 * one fp32 scale per 128x128 block, with two-level accumulation: the FP8
 * products of each 128-wide K block are summed on the tensor cores and then
 * promoted into an fp32 accumulator with both scales applied.
 *
 * Sources for the operation:
 *   - "DeepGEMM" overview (zixun.chuxinyishu.com/article/345.html), section
 *     "FP8与细粒度缩放": FP8 operands, activations scaled per slice, weights
 *     per matrix block, higher-precision accumulation; section "约300行JIT核心"
 *     paragraph on contiguous and masked MoE layouts (grouping along M, the
 *     masked layout meeting the communication library); section "swapAB与
 *     Mega MoE": computing the transposed product for thin M.
 *   - "一文看懂 DeepSeek 開源項目第三彈" (animattoys.com), sections
 *     "為現代 AI 計算而造" and "DeepGEMM 部署指南": normal and MoE grouped
 *     GEMM, two-level accumulation (promotion) because FP8 tensor-core
 *     accumulation is imprecise.
 *   - DeepSeek-V3 review "28.5 倍压缩 + 1/10 成本"
 *     (developer.cloud.tencent.cn/article/2686109), "创新之处" item 4: one
 *     scale per 128 elements, 128x128 block scaling; "风险与不足" item 6: the
 *     448.0 FP8 bound used by the quantizer.
 *
 * Conventions shared by every entry point:
 *   - All data pointers are DEVICE pointers allocated and owned by the caller.
 *     The library never allocates, frees or retains them.
 *   - Every data pointer must be 16-byte aligned (TMA requirement).
 *   - Calls are asynchronous on `stream` (NULL = legacy default stream). The
 *     host returns after the launch; nothing synchronises the host.
 *   - e4m3 payloads are bytes (OCP E4M3 "fn": bias 7, no infinities, max 448).
 *     bf16 tensors are passed as their 16-bit patterns. Scales are fp32.
 *   - Argument errors are reported synchronously (FG_ERR_INVALID_ARG or
 *     FG_ERR_UNSUPPORTED) and then nothing is launched. Launch failures
 *     return FG_ERR_CUDA. Faults detected on the device (a bounded wait that
 *     gave up, masked_m outside [0, M_max], an m_indices entry >= G) set a
 *     device status word read by fg_get_device_status(); the kernels never
 *     trap and never wait without a bound.
 *   - fg_last_error() returns a human-readable detail of the last failing
 *     call on the calling host thread.
 *
 * Scale layouts:
 *   - Activation scales (SFA) are "MN-major": for each K block kb the scales
 *     of all M rows are contiguous, with a row stride of fg_sfa_stride(M) =
 *     round_up(M, 4) floats so that every K block starts 16-byte aligned:
 *       sfa[(g * (K/128) + kb) * fg_sfa_stride(M) + m]
 *     (g = group of a batched quantizer call / expert of the masked layout;
 *     0 otherwise). Entries m in [M, stride) are padding and never read.
 *   - Weight scales (SFB): sfb[(g * ceil(N/128) + nb) * (K/128) + kb].
 */
#ifndef FP8GEMM_H_
#define FP8GEMM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as the CUDA runtime's cudaStream_t. */
struct CUstream_st;
typedef struct CUstream_st* cudaStream_t;

typedef enum {
  FG_OK = 0,
  FG_ERR_INVALID_ARG = 1,  /* bad size, null or misaligned pointer */
  FG_ERR_UNSUPPORTED = 2,  /* valid request this build does not cover */
  FG_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
  FG_ERR_DEVICE = 4        /* device status word set (see fg_get_device_status) */
} fg_status;

/* Device status word values (returned through fg_get_device_status). */
#define FG_DEVICE_OK 0
#define FG_DEVICE_WAIT_TIMEOUT 1   /* a bounded pipeline wait gave up */
#define FG_DEVICE_BAD_MASKED_M 2   /* masked_m[e] < 0 or > M_max (clamped) */
#define FG_DEVICE_BAD_M_INDEX 3    /* m_indices entry >= G (tile skipped) */
#define FG_DEVICE_BAD_K_GROUP 4    /* ks entry < 0, not a multiple of 128, or sum > T (truncated) */
#define FG_DEVICE_BAD_SCALE 5      /* a block-scaled _ue8m0 GEMM read a scale that is not a power of two */
#define FG_DEVICE_EP_OVERFLOW 6    /* a local expert received more than M_max rows (the rest dropped) */

/* Row stride (in floats) of the MN-major activation-scale layout. */
int fg_sfa_stride(int M);

/*
 * Activation quantizer (per token, per 128-channel slice).
 * For every group g < num_groups, row m < M and K block kb:
 *   amax  = max |x[g][m][kb*128 .. kb*128+127]|  (bf16 widened exactly)
 *   amx   = max(amax, 1e-4f)
 *   sfa   = amx / 448.0f                         (fp32, IEEE division)
 *   q[..] = e4m3_rne_satfinite(x[..] * (448.0f / amx))  (fp32 product)
 * x: bf16 [num_groups][M][K]; q: e4m3 [num_groups][M][K];
 * sfa: fp32, MN-major layout above, num_groups * (K/128) * fg_sfa_stride(M)
 * floats. K % 128 == 0, M >= 0, num_groups >= 1. The masked layout's A is
 * one call with num_groups = G, M = M_max; the dense and contiguous A is one
 * call with num_groups = 1.
 */
fg_status per_token_cast_to_fp8(const uint16_t* x, uint8_t* q, float* sfa, int num_groups,
                                int M, int K, cudaStream_t stream);

/*
 * Weight quantizer (per 128x128 block). Same arithmetic with amax over each
 * block of 128 rows x 128 columns; a last block along N that has fewer than
 * 128 rows uses only its valid rows.
 * x: bf16 [num_groups][N][K]; q: e4m3 [num_groups][N][K];
 * sfb: fp32 [num_groups][ceil(N/128)][K/128]. K % 128 == 0, N >= 1.
 */
fg_status per_block_cast_to_fp8(const uint16_t* x, uint8_t* q, float* sfb, int num_groups,
                                int N, int K, cudaStream_t stream);

/*
 * The same two quantizers with power-of-two scales (the UE8M0 scale format of
 * DeepSeek-V3.1; DeepSeek-V3 review "28.5 倍压缩 + 1/10 成本", "创新之处"
 * item 4: scales quantized to powers of two, so a shift replaces a multiply):
 *   scale = the smallest power of two at or above max(amax, 1e-4f) / 448
 *           (from the fp32 bits of the quotient)
 *   q     = e4m3_rne_satfinite(x / scale)   (exact: no element exceeds 448)
 * Layouts, sizes and errors as for the fp32-scale forms above; the scales are
 * written as fp32 values, so every GEMM entry point accepts them.
 */
fg_status per_token_cast_to_fp8_ue8m0(const uint16_t* x, uint8_t* q, float* sfa, int num_groups,
                                      int M, int K, cudaStream_t stream);
fg_status per_block_cast_to_fp8_ue8m0(const uint16_t* x, uint8_t* q, float* sfb, int num_groups,
                                      int N, int K, cudaStream_t stream);

/*
 * Weight dequantization, the third kernel of the FP8 quantize / dequantize /
 * GEMM trio (DeepSeek-V3 review "28.5 倍压缩 + 1/10 成本", "创新之处" item 4
 * and "可复用的模式与技巧" item 3). For every group g, row n and column k:
 *   x[g][n][k] = bf16( fp32( e4m3(q[g][n][k]) * sfb[g][n/128][k/128] ) )
 * the fp32 product and the bf16 conversion both round to nearest even; NaN
 * codes give NaN. q: e4m3 [num_groups][N][K]; sfb: fp32
 * [num_groups][ceil(N/128)][K/128] (the layout per_block_cast_to_fp8 writes);
 * x: bf16 [num_groups][N][K]. K % 128 == 0, N >= 1, num_groups >= 1.
 */
fg_status per_block_dequant_to_bf16(const uint8_t* q, const float* sfb, uint16_t* x,
                                    int num_groups, int N, int K, cudaStream_t stream);

/*
 * Dense FP8 GEMM, "NT": D[m][n] = sum_kb sa[m][kb] * sb[n/128][kb] *
 *   sum_{k in kb} e4m3(A[m][k]) * e4m3(B[n][k]), rounded once to bf16.
 * A: e4m3 [M][K] (row-major, K contiguous); sfa: MN-major [K/128][stride(M)];
 * B: e4m3 [N][K]; sfb: [ceil(N/128)][K/128]; D: bf16 [M][N] row-major.
 * M >= 0, N >= 16 with N % 16 == 0, K % 128 == 0.
 * For M <= 64 the library uses the swapped product D^T = B * A^T so that the
 * thin token dimension lands on the tensor-core instruction's N side, and
 * when that leaves most SMs idle it splits K across the 2 or 4 CTAs of a
 * thread-block cluster, which sum their partials through distributed shared
 * memory in a fixed order (deterministic; no scratch memory is used).
 */
fg_status fp8_gemm_nt(const uint8_t* A, const float* sfa, const uint8_t* B, const float* sfb,
                      uint16_t* D, int M, int N, int K, cudaStream_t stream);

/*
 * MoE grouped FP8 GEMM, contiguous layout: the token groups of G experts are
 * stacked along M, each group starting on a 128-row boundary and padded to a
 * multiple of 128 rows. Row m uses expert m_indices[m]'s weights; padding
 * rows carry m_indices[m] = -1 (their A rows should be zero).
 * A: e4m3 [M_total][K]; sfa: MN-major [K/128][stride(M_total)];
 * B: e4m3 [G][N][K]; sfb: [G][ceil(N/128)][K/128]; D: bf16 [M_total][N];
 * m_indices: int32 [M_total], device memory.
 * Contract: all valid rows of a 128-row block share one expert and come
 * before its padding rows. D rows with m_indices[m] = -1 are not written.
 * M_total % 128 == 0, G >= 1, N % 16 == 0, K % 128 == 0.
 */
fg_status fp8_grouped_gemm_contiguous(const uint8_t* A, const float* sfa, const uint8_t* B,
                                      const float* sfb, uint16_t* D, const int32_t* m_indices,
                                      int M_total, int N, int K, int G, cudaStream_t stream);

/*
 * MoE grouped FP8 GEMM, masked layout: expert e owns an M_max-row slab of A
 * and D, of which the first masked_m[e] rows are valid. masked_m stays on the
 * device and is never read by the host, so the call does not synchronise.
 * A: e4m3 [G][M_max][K]; sfa: MN-major [G][K/128][stride(M_max)];
 * B: e4m3 [G][N][K]; sfb: [G][ceil(N/128)][K/128]; D: bf16 [G][M_max][N];
 * masked_m: int32 [G], device memory. expected_m: host-side hint of the
 * typical masked_m (selects the tile shape; any value is correct).
 * D rows m >= masked_m[e] are not written and the kernel does not read the
 * A rows past masked_m[e] into any stored output.
 * G >= 1, M_max >= 1, N % 16 == 0, K % 128 == 0.
 */
fg_status fp8_grouped_gemm_masked(const uint8_t* A, const float* sfa, const uint8_t* B,
                                  const float* sfb, uint16_t* D, const int32_t* masked_m, int G,
                                  int M_max, int N, int K, int expected_m, cudaStream_t stream);

/*
 * The three GEMMs above for power-of-two scales (the UE8M0 scale format;
 * DeepSeek-V3 review "28.5 倍压缩 + 1/10 成本", "创新之处" item 4: scales
 * quantized to powers of two so that applying one is a shift). Same operation,
 * arguments, layouts, contracts and errors as fp8_gemm_nt,
 * fp8_grouped_gemm_contiguous and fp8_grouped_gemm_masked; additionally every
 * sfa and sfb entry that is read must be a power of two in the fp32 normal
 * range (what per_token_cast_to_fp8_ue8m0 / per_block_cast_to_fp8_ue8m0
 * write), or zero (which acts as 2^-127). The block-scaled kernel keeps only
 * each scale's exponent field; it checks every weight scale it reads and the
 * token scales of every row it stores, and a scale with a sign or mantissa
 * bit set, or an infinite or NaN scale, sets FG_DEVICE_BAD_SCALE: the call's
 * output is then not the product of the given scales and must be discarded.
 * (The promoted kernel that thin shapes use applies any fp32 scale exactly
 * and checks nothing.)
 *
 * For token tiles of 128 rows (or pairs of them of one expert, computed by
 * the two CTAs of a cluster) the scales are applied inside the tensor core (tcgen05.mma
 * kind::mxf8f6f4.block_scale, one UE8M0 scale per row per 32 K elements), and
 * the whole K range accumulates in tensor memory in fp32 with no promotion
 * pass; the products a * b * sa * sb are exact, only the order of
 * the fp32 additions differs from the promoted form. Thin shapes (dense
 * M <= 64, masked expected_m <= 64) run the promoted swapped kernel, which is
 * exact per K block for power-of-two scales as well.
 */
fg_status fp8_gemm_nt_ue8m0(const uint8_t* A, const float* sfa, const uint8_t* B,
                            const float* sfb, uint16_t* D, int M, int N, int K,
                            cudaStream_t stream);
fg_status fp8_grouped_gemm_contiguous_ue8m0(const uint8_t* A, const float* sfa, const uint8_t* B,
                                            const float* sfb, uint16_t* D,
                                            const int32_t* m_indices, int M_total, int N, int K,
                                            int G, cudaStream_t stream);
fg_status fp8_grouped_gemm_masked_ue8m0(const uint8_t* A, const float* sfa, const uint8_t* B,
                                        const float* sfb, uint16_t* D, const int32_t* masked_m,
                                        int G, int M_max, int N, int K, int expected_m,
                                        cudaStream_t stream);

/*
 * MoE expert FFN with power-of-two scales: for every expert e,
 *   GU = bf16(X_e W1_e^T)          (first grouped GEMM; W1_e has 2I rows: I gate
 *                                   rows, then I up rows)
 *   h  = bf16(silu(gate) * up)     (silu(g) = g / (1 + exp(-g)) in fp32, exp by a
 *                                   fixed Cody-Waite + degree-7 Taylor sequence)
 *   Hq, sfh = per_token_cast_to_fp8_ue8m0(h)
 *   Y  = bf16(Hq W2_e^T)           (second grouped GEMM; W2_e is H x I)
 * the single-GPU part of the "Mega MoE" kernel, which fuses both expert GEMMs
 * with the SwiGLU activation in one kernel ("DeepGEMM" overview, section
 * "swapAB与Mega MoE"). The first GEMM's tiles run the SwiGLU and the
 * requantization in their epilogue (no bf16 intermediate goes to memory).
 * For decode-sized batches (at most 128 expected rows per expert) one
 * persistent launch computes both GEMMs: the first GEMM's tiles count up a
 * ready counter per 128-token tile once its quantized activations are
 * written; the second GEMM's tiles come after them in every CTA's work list
 * and wait (bounded) for their token tile's counter, so the second GEMM starts
 * on finished token tiles while the first GEMM's last tiles still run, with no
 * second launch. Larger batches run the two GEMMs as two launches, which is
 * faster there (see fg_set_ffn_mode).
 * Scales must be powers of two (as for the _ue8m0 GEMMs).
 * Contiguous: X e4m3 [M_total][H], sfx MN-major [H/128][stride(M_total)],
 *   m_indices int32 [M_total] (contract of fp8_grouped_gemm_contiguous);
 *   Hq e4m3 [M_total][I], sfh [I/128][stride(M_total)], Y bf16 [M_total][H].
 * Masked: X [G][M_max][H], sfx [G][H/128][stride(M_max)], masked_m int32 [G];
 *   Hq [G][M_max][I], sfh [G][I/128][stride(M_max)], Y [G][M_max][H].
 * W1 e4m3 [G][2I][H], sfw1 [G][2I/128][H/128]; W2 e4m3 [G][H][I],
 * sfw2 [G][H/128][I/128]. GU: optional (NULL = not written) bf16 [rows][2I]
 * output of the first GEMM (gate columns, then up columns), which the SwiGLU
 * backward pass needs. Hq, sfh and Y (and GU) are written on valid rows only.
 * ws: device workspace of at least fg_moe_ffn_workspace_bytes(layout, M, G)
 *   bytes (M = M_total or M_max), 16-byte aligned, owned by the caller, for
 *   the ready counters of the one-launch form (required for both forms); the
 *   call clears the counters it uses (cudaMemsetAsync on `stream`) before its
 *   kernel, so the workspace needs no initialisation, and two calls in flight
 *   at once must not share it. Smaller: FG_ERR_INVALID_ARG.
 * H % 128 == 0, I % 128 == 0, G >= 1; other limits as for the grouped GEMMs.
 */
#define FG_LAYOUT_CONTIGUOUS 0
#define FG_LAYOUT_MASKED 1
/* Form of the expert FFN (process-wide): 0 = automatic (one launch when the
 * expected rows per expert, expected_m or M_total / G, are at most 128, else
 * two launches), 1 = always one launch, 2 = always two launches. Other
 * values: FG_ERR_INVALID_ARG. */
fg_status fg_set_ffn_mode(int mode);
/* Workspace bytes of the expert FFN (0 for invalid arguments). */
size_t fg_moe_ffn_workspace_bytes(int layout, int M, int G);
fg_status fp8_moe_ffn_contiguous_ue8m0(const uint8_t* X, const float* sfx, const uint8_t* W1,
                                      const float* sfw1, const uint8_t* W2, const float* sfw2,
                                      uint8_t* Hq, float* sfh, uint16_t* GU, uint16_t* Y,
                                      const int32_t* m_indices, int M_total, int H, int I, int G,
                                      void* ws, size_t ws_bytes, cudaStream_t stream);
fg_status fp8_moe_ffn_masked_ue8m0(const uint8_t* X, const float* sfx, const uint8_t* W1,
                                  const float* sfw1, const uint8_t* W2, const float* sfw2,
                                  uint8_t* Hq, float* sfh, uint16_t* GU, uint16_t* Y,
                                  const int32_t* masked_m, int G, int M_max, int H, int I,
                                  int expected_m, void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * The masked expert FFN above in its one-launch form, for callers that must
 * not allocate device memory: it takes no workspace. This entry point has no
 * counterpart in the pages; it exists for code that is handed its input and
 * output buffers but cannot obtain more device memory - for example a serving
 * runtime that reserves all of the GPU's memory for its weights and KV cache
 * when it starts and hands each operator fixed buffers, or a plugin that runs
 * inside another framework's memory manager and is given no allocator - so
 * that a workspace would otherwise have to be carved out of someone else's
 * buffers.
 * Its ready counters live in a fixed array of this library's own device
 * memory (16 KB, 4096 counters; every GPU that loads the library holds it
 * until the process exits). The call allocates and frees nothing; it clears
 * the counters it uses (cudaMemsetAsync on `stream`) before its kernel.
 * Limit: G * ceil(M_max / 128) <= 4096 token tiles; larger problems return
 * FG_ERR_UNSUPPORTED (use fp8_moe_ffn_masked_ue8m0 with a workspace).
 * The first call on a device looks up the array's device address there
 * (once, cached); make that first call before capturing any stream.
 * All calls share the one array per device: calls whose kernels can overlap
 * on the GPU (on different streams) race on it and give wrong results;
 * calls in order on one stream are safe.
 * Arguments, layouts, results and other errors: those of
 * fp8_moe_ffn_masked_ue8m0 (always the one-launch form).
 */
fg_status fp8_moe_ffn_masked_ue8m0_noalloc(const uint8_t* X, const float* sfx, const uint8_t* W1,
                                          const float* sfw1, const uint8_t* W2, const float* sfw2,
                                          uint8_t* Hq, float* sfh, uint16_t* GU, uint16_t* Y,
                                          const int32_t* masked_m, int G, int M_max, int H, int I,
                                          int expected_m, cudaStream_t stream);

/*
 * K-grouped GEMM with power-of-two scales, for the weight gradients of MoE
 * experts in FP8 training (dW_e = dY_e^T X_e: the contraction runs over the
 * tokens routed to each expert). The experts' token ranges are stacked along
 * K; both operands carry one scale per row per 128-token block:
 *   D[e][m][n] = sum over expert e's token blocks tb of
 *                sa[m][tb] * sb[n][tb] * sum_{t in tb} a[m][t] * b[n][t],
 * accumulated in fp32 (block-scaled tensor-core MMAs, whole range in tensor
 * memory). Sources: FP8 training among DeepGEMM's uses ("一文看懂 DeepSeek
 * 開源項目第三彈", section "為現代 AI 計算而造") and per-128-element scaling
 * of every GEMM operand (DeepSeek-V3 review, "创新之处" item 4).
 * A: e4m3 [M][T] (K contiguous); sfa: fp32 MN-major [T/128][stride(M)]
 * (the layout per_token_cast_to_fp8_ue8m0 writes for a [M][T] input);
 * B: e4m3 [N][T]; sfb: fp32 MN-major [T/128][stride(N)]; D: fp32 [G][M][N];
 * ks: int32 [G] device array of token counts, each a multiple of 128 and
 * summing to T (violations set FG_DEVICE_BAD_K_GROUP; the counts are then
 * truncated). An expert with ks[e] = 0 gets D[e] = 0. Scales must be powers of
 * two. G >= 1, M >= 1, N % 16 == 0, T % 128 == 0 (T = 0 allowed).
 */
fg_status fp8_k_grouped_gemm_nt_ue8m0(const uint8_t* A, const float* sfa, const uint8_t* B,
                                     const float* sfb, float* D, const int32_t* ks, int G, int M,
                                     int N, int T, cudaStream_t stream);

/*
 * Expert-parallel dispatch into the masked layout and the combine after it,
 * around an all-to-all exchange that the caller performs (NCCL over
 * NVLink); the masked layout is the one the grouped GEMM shares with the
 * communication library ("DeepGEMM" overview, section "约300行JIT核心",
 * paragraph on MoE layouts; the transfer over NVLink: section "swapAB与Mega
 * MoE"). E experts over W GPUs, G = E / W local experts per GPU: GPU d holds
 * experts [d * G, (d + 1) * G). A "pair" is (token t, choice j), p = t * k + j,
 * with expert topk_idx[p]. All arrays are device arrays owned by the caller.
 *
 * ep_dispatch_layout: counts[E] = pairs of each expert; send_pos[T * k] = the
 *   pair's row in the send buffer, in which pairs are ordered by expert, and
 *   within an expert by p (so GPU d's pairs are the contiguous rows
 *   [sum of counts of experts < d * G, + its experts' counts)). A negative
 *   expert is a dropped choice (send_pos = -1); an expert >= E too, and it
 *   sets FG_DEVICE_BAD_M_INDEX. T >= 0, k >= 1, E >= 1.
 * ep_dispatch_pack: copies token row t of q (e4m3 [T][K]) and its K / 128
 *   scales (MN-major sfa [K/128][stride(T)], what per_token_cast_to_fp8
 *   writes) to row send_pos[p] of send_q [P][K] and send_s [P][K/128] for
 *   every pair with send_pos >= 0 (P = counts summed, at most T * k).
 * ep_dispatch_unpack_masked: the R received rows (recv_q [R][K], recv_s
 *   [R][K/128]) come source GPU by source GPU, each source's rows local expert
 *   by local expert, recv_counts[s * G + g] of them (int32, device) - the
 *   segments the sources' layouts put in front of this GPU. Row i of (s, g)
 *   goes to slot (rows of expert g from sources before s) + i of the masked
 *   layout A [G][M_max][K], sfa [G][K/128][stride(M_max)]; masked_m[g] = rows
 *   of g (capped at M_max: rows past it are dropped, recv_slot = -1 and
 *   FG_DEVICE_EP_OVERFLOW); recv_slot[r] = g * M_max + slot. W * G <= 4096.
 * ep_combine_gather: out[r] = D row recv_slot[r] (bf16 [.][N] -> [R][N], zero
 *   for dropped rows): the masked GEMM's outputs back in receive order, to be
 *   sent back to their sources. N % 8 == 0.
 * ep_combine_reduce: with y [P][N] the rows returned in send order,
 *   out[t][n] = bf16(sum over j = 0..k-1 of topk_w[t][j] * y[send_pos[t*k+j]][n]),
 *   each term an fp32 fused multiply-add in j order, rounded to nearest even
 *   once; choices with send_pos < 0 add nothing. N % 8 == 0.
 * Errors: FG_ERR_INVALID_ARG for sizes and null or misaligned pointers.
 */
fg_status ep_dispatch_layout(const int32_t* topk_idx, int T, int k, int E, int32_t* counts,
                             int32_t* send_pos, cudaStream_t stream);
fg_status ep_dispatch_pack(const uint8_t* q, const float* sfa, const int32_t* send_pos, int T, int k,
                           int K, uint8_t* send_q, float* send_s, cudaStream_t stream);
fg_status ep_dispatch_unpack_masked(const uint8_t* recv_q, const float* recv_s,
                                    const int32_t* recv_counts, int W, int G, int R, int M_max,
                                    int K, uint8_t* A, float* sfa, int32_t* masked_m,
                                    int32_t* recv_slot, cudaStream_t stream);
fg_status ep_combine_gather(const uint16_t* D, const int32_t* recv_slot, int R, int N, uint16_t* out,
                            cudaStream_t stream);

/*
 * The same dispatch with a fixed capacity of C rows per destination GPU, so
 * that every exchange has equal, host-known split sizes (C rows to and from
 * every GPU) and no count has to be read back to the host before it: the
 * whole layer then runs without a host synchronisation. Not a step the pages
 * name; it trades exchange bytes (W * C rows each way) for that.
 * ep_dispatch_layout_capacity: as ep_dispatch_layout, with W GPUs of
 *   G = E / W experts each (E % W == 0), but send_pos[p] = d * C + (the
 *   pair's position among destination d's pairs, ordered by expert, then by
 *   p), d = expert / G; a pair whose position would be C or more is dropped
 *   (send_pos = -1, FG_DEVICE_EP_OVERFLOW), and counts[e] counts only the
 *   pairs of expert e that are sent (what the receivers must expect). The send buffers of
 *   ep_dispatch_pack then need W * C rows (rows a destination does not fill
 *   are left as they were and never read).
 * ep_dispatch_unpack_masked_capacity: as ep_dispatch_unpack_masked for a
 *   receive buffer of W * C rows in which source s's rows start at row s * C
 *   (local expert by local expert, recv_counts[s * G + g] of them); the rows
 *   after a source's last one get recv_slot = -1. recv_slot holds W * C
 *   entries; counts that put more than C rows in a segment set
 *   FG_DEVICE_EP_OVERFLOW. ep_combine_gather and ep_combine_reduce are used
 *   unchanged with R = W * C and these send_pos.
 * C >= 1, W * C < 2^31; other errors as above.
 */
fg_status ep_dispatch_layout_capacity(const int32_t* topk_idx, int T, int k, int E, int W, int C,
                                      int32_t* counts, int32_t* send_pos, cudaStream_t stream);
fg_status ep_dispatch_unpack_masked_capacity(const uint8_t* recv_q, const float* recv_s,
                                             const int32_t* recv_counts, int W, int G, int C, int M_max,
                                             int K, uint8_t* A, float* sfa, int32_t* masked_m,
                                             int32_t* recv_slot, cudaStream_t stream);
fg_status ep_combine_reduce(const uint16_t* y, const int32_t* send_pos, const float* topk_w, int T, int k,
                            int N, uint16_t* out, cudaStream_t stream);

/*
 * Tuning knob of the three _ue8m0 GEMMs (process-wide). width = 0: choose the
 * tile per shape (default). Otherwise always use the block-scaled kernel, thin
 * shapes included, with weight tiles of `width` rows: 128, 224 or 256 with
 * pair = 0 (one CTA per 128-token tile), or 224 or 192 with pair = 1 (two CTAs
 * of a cluster per pair of token tiles of one expert, tcgen05 cta_group::2).
 * Other values: FG_ERR_INVALID_ARG.
 */
fg_status fg_set_ue8m0_tile(int width, int pair);

/*
 * Synchronises `stream`, then reads and clears the device status word of the
 * current device. Returns FG_OK when it was clear, FG_ERR_DEVICE otherwise
 * (the detail is in fg_last_error and *code, which may be NULL).
 * There is one status word per device, shared by every stream and every call
 * of this library on that device: it holds the first FG_DEVICE_* code any
 * kernel recorded since it was last cleared. Only `stream` is synchronised,
 * so a call still running on another stream may set the word after it was
 * read; to attribute a status to one call, run that call alone (or
 * synchronise the device) before this read.
 */
fg_status fg_get_device_status(cudaStream_t stream, int* code);

/*
 * Self-test of the bounded wait used by every pipeline barrier: launches one
 * CTA that waits on a barrier nobody arrives at, for at most timeout_us
 * microseconds, after which it sets FG_DEVICE_WAIT_TIMEOUT and returns.
 */
fg_status fg_selftest_wait_timeout(int timeout_us, cudaStream_t stream);

/*
 * Tensor-core rate (a measurement aid, not a step of the method): the FP8
 * tensor-core instruction every GEMM here issues (tcgen05.mma kind::f8f6f4,
 * M = 128, N = 256, K = 32), run back to back from operands that stay in
 * shared memory, with nothing loaded or promoted, so that the time of a
 * launch gives the rate the tensor cores sustain at the clock of the moment.
 * The GEMMs are judged by their FP8 TFLOPS ("DeepGEMM" overview, section
 * "约300行JIT核心"); this gives the ceiling of that figure on this GPU.
 *
 * One CTA on each of the fg_fp8_mma_peak_ctas() SMs; each runs `iters` K
 * blocks of 128 (1 <= iters <= 32768), i.e. 2 * 128 * 256 * 128 * iters
 * FLOPs per CTA. The operands are generated in the kernel from small
 * integers, so the result is exact and shows that every MMA ran:
 *   out[c][m][n] = iters * 8 * sum_{j<16} A(m, j) * B(n, j),
 *   A(m, j) = (2m + 3j) mod 5 - 2,  B(n, j) = (3n + 2j + floor(n/16)) mod 5 - 2,
 * for every CTA c < fg_fp8_mma_peak_ctas(), m < 128, n < 256.
 * out: device fp32 [fg_fp8_mma_peak_ctas()][128][256], caller-owned.
 * Errors: FG_ERR_INVALID_ARG (iters out of range, null out),
 * FG_ERR_UNSUPPORTED / FG_ERR_CUDA as for the GEMMs.
 */
int fg_fp8_mma_peak_ctas(void); /* SM count of the current device; 0 if it is not usable */
fg_status fg_fp8_mma_peak(int iters, float* out, cudaStream_t stream);

const char* fg_status_string(fg_status s);
const char* fg_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8GEMM_H_ */
