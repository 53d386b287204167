/*
 * qgemm.h — C ABI of the B200 (sm_100a) quantized linear-layer GEMM library
 * (libqgemm.so).
 *
 * The library computes, on one GPU,
 *
 *     y[M, N] = dequant(A_q)[M, K] . dequant(W_q)[N, K]^T      (bf16 out)
 *
 * for the 8-bit formats of the vLLM linear backend described in "Helion in
 * the vLLM backend: one GEMM, tuning per shape" (ai-radar.it; first
 * paragraph: FP8_Dynamic, W8A8_INT8, Block_FP8) and for NVFP4, the format of
 * FlashInfer's mm_fp4 GEMM (FlashInfer PR 3948, "perf(gemm): update mm_fp4
 * cute-dsl tactic heuristic ...", benchmark command with --use_nvfp4 and
 * --use_128x4_sf_layout).  One kernel family covers the three algorithms of
 * the same article (second paragraph): Standard, Split-K (power-of-two
 * splits up to 256, third paragraph) and Swap-AB, computed as
 * (W_q . A_q^T)^T so that the weight rows fill the 128-row MMA slot.  An
 * ahead-of-time table maps (format, M, N, K) to a configuration (third and
 * fourth paragraphs; M is bucketed as in FlashInfer PR 3948, "M bucketing by
 * floor(log2 M)").
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers unless a parameter says
 *     otherwise.  The caller owns every buffer, the workspace and the stream;
 *     the run path (qgemm_quantize_act, qgemm_run, qgemm_dispatch) allocates
 *     nothing, synchronises nothing and copies nothing between host and
 *     device, so it may be captured into a CUDA graph.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy stream).
 *   - Arguments are checked on the host before any launch; a failed check
 *     returns a status and launches nothing.  Zero-sized M, N or K is
 *     QG_ERR_INVALID_ARG (FlashInfer PR 3948 review: guard against
 *     zero-dimension inputs).
 *   - Row-major everywhere; "K-contiguous" means element (r, k) of a
 *     [rows, K] operand is at byte r * row_bytes + k * elem_bytes.
 *   - Device memory alignment: every pointer 16-byte aligned.
 */
#ifndef QGEMM_H_
#define QGEMM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QGEMM_ABI_VERSION 1

typedef enum {
  QG_FP8_DYNAMIC = 0, /* e4m3 codes, fp32 scale per token / per channel        */
  QG_W8A8_INT8 = 1,   /* int8 codes, fp32 scale per token / per channel        */
  QG_BLOCK_FP8 = 2,   /* e4m3 codes, fp32 scale per 1x128 act group / 128x128 W block */
  QG_NVFP4 = 3        /* e2m1 codes, e4m3 scale per 16 K elements + fp32 tensor scale */
} qg_format;

typedef enum {
  QG_OK = 0,
  QG_ERR_INVALID_ARG = 1,    /* null pointer, bad size, misaligned pointer, bad enum   */
  QG_ERR_UNSUPPORTED = 2,    /* shape/config the kernels do not cover, or not sm_100   */
  QG_ERR_WORKSPACE = 3,      /* workspace missing or smaller than *_workspace_size     */
  QG_ERR_TABLE_IO = 4,       /* table file missing, corrupt or of another version      */
  QG_ERR_TABLE_MISS = 5,     /* (reserved) strict dispatch found no entry              */
  QG_ERR_CUDA = 6,           /* a CUDA runtime/driver call or a launch failed          */
  QG_ERR_DEVICE_TIMEOUT = 7, /* a bounded in-kernel wait expired (qgemm_device_error)  */
  QG_ERR_NO_DEVICE = 8       /* no CUDA device visible                                 */
} qg_status;

/* Output kind of qgemm_run. */
typedef enum {
  QG_OUT_BF16 = 0, /* y as bf16 [M, ldy]                                            */
  QG_OUT_ACC = 1   /* debug: the raw contraction before the scale epilogue, [M, ldy]:
                      int32 for W8A8_INT8 (exact), fp32 for the other formats (for
                      Block_FP8 this is the group-promoted sum, i.e. the final y
                      before bf16 rounding)                                         */
} qg_out_kind;

/* Kernel configuration: which kernel runs (variant) and its tunables. */
typedef struct {
  int32_t split_k;     /* 1, 2, 4, ..., 256: K is cut into split_k slices of whole
                          128-byte K tiles, each reduced by its own CTA            */
  int32_t swap_ab;     /* 1: weights take the 128-row MMA operand and tokens the
                          N operand (y^T = W_q A_q^T); 0: tokens take the 128 rows */
  int32_t tile_n;      /* MMA N extent: tokens per CTA when swap_ab = 1, weight
                          rows per CTA when swap_ab = 0; one of 16,32,64,128,256   */
  int32_t stages;      /* shared-memory pipeline depth, 2..12 (capped by smem)     */
  int32_t reduce_mode; /* split_k > 1 only; every mode sums the partials in split
                          order, so all three give identical bits:
                          0 = the split_k CTAs of a tile form a thread-block
                              cluster and sum through distributed shared memory
                              (split_k <= 8, no workspace);
                          1 = partials in the workspace + a second-pass kernel;
                          2 = partials in the workspace, summed in-kernel by the
                              last-arriving CTA of each tile (tile counters)    */
  int32_t variant;     /* 0: the tile kernel (tcgen05, the fields above);
                          1: the decode ("skinny") kernel for FP8_DYNAMIC,
                          W8A8_INT8 and BLOCK_FP8: warp-level MMAs with register
                          accumulators, each CTA owning `rows` weight rows over
                          the whole of K and tile_n (8, 16 or 32) tokens;
                          requires split_k = 1, swap_ab = 1, reduce_mode = 0,
                          and `stages` (the ring of 128-byte K tiles, 2..64) a
                          multiple of the K groups of its eight compute warps:
                          64 / rows (128 / rows for tile_n = 8);
                          2: the persistent kernel for the 8-bit formats at
                          large M: one CTA per SM walks the 128 x tile_n
                          output tiles, so a tile's epilogue (bf16 through TMA
                          stores) overlaps the next tile's MMAs (FP8_DYNAMIC,
                          W8A8_INT8: two TMEM accumulators; BLOCK_FP8: the
                          promotion's group buffers, free once a tile's last
                          group is promoted); requires split_k = 1, swap_ab = 0,
                          reduce_mode = 0, rows = 0, tile_n 128 or 256,
                          stages 2..12 (capped by shared memory), and bf16
                          output (QG_ERR_UNSUPPORTED otherwise); y is bitwise
                          that of variant 0 with the same tile_n;
                          3: BLOCK_FP8 on CTA pairs at medium and large M:
                          clusters of two CTAs (one per SM) walk output
                          tiles of 256 tokens x tile_n channels; each CTA
                          loads its 128 token rows and tile_n / 2 of the
                          weight rows, the even CTA issues one cta_group::2
                          MMA (M = 256) per K step, and each CTA promotes its
                          own rows through 512 / tile_n TMEM group buffers;
                          requires split_k = 1, swap_ab = 0, reduce_mode = 0,
                          rows = 0, tile_n 128 or 256, stages 2..12 (capped
                          by shared memory), bf16 output and an output row
                          pitch of a multiple of 8 elements
                          (QG_ERR_UNSUPPORTED otherwise); y is bitwise that
                          of variant 0 with the same tile_n                  */
  int32_t rows;        /* variant 1: weight rows per CTA, 8, 16, 32 or 64 (at
                          least 16 for tile_n = 8); variants 0, 2, 3: 0       */
  int32_t reserved;    /* must be zero                                            */
} qg_config;

/* A quantized operand (activations A_q or weights W_q); non-owning views.
 * Layouts by format, for an operand of `rows` rows and K reduction elements:
 *   q:     FP8_DYNAMIC, BLOCK_FP8: e4m3 bytes [rows, K]
 *          W8A8_INT8: int8 [rows, K]
 *          NVFP4: packed e2m1 [rows, K/2] bytes, element 2j in the low nibble
 *   scale: FP8_DYNAMIC, W8A8_INT8: fp32 [rows]
 *          BLOCK_FP8 activations: fp32 [rows, K/128]
 *          BLOCK_FP8 weights:     fp32 [ceil(rows/128), K/128]
 *          NVFP4: e4m3 block scales in the 128x4 tiled layout: the
 *                 [rows, K/16] scale matrix is padded to R = ceil(rows/128)*128
 *                 rows and C = ceil(K/256)*16 columns and cut into 128x4
 *                 atoms of 512 bytes; atom (rb, cb) starts at byte
 *                 (rb * C/4 + cb) * 512 and holds scale (r, c) at
 *                 (r%32)*16 + ((r%128)/32)*4 + c%4.  Padding bytes are 0.
 *   global_scale: NVFP4 only — device fp32 scalar g (decode scale of the
 *                 tensor: x ~= dec(code) * dec(block scale) * g).          */
typedef struct {
  void* q;
  void* scale;
  float* global_scale;
  int32_t rows;
  int32_t K;
} qg_operand;

/* ---------------------------------------------------------------- sizes -- */

/* Bytes of the `q` and `scale` buffers of an operand (weights when
 * is_weight != 0).  Returns QG_ERR_INVALID_ARG for an unknown format or
 * non-positive sizes. */
qg_status qgemm_operand_bytes(qg_format f, int is_weight, int rows, int K,
                              size_t* q_bytes, size_t* scale_bytes);

/* Scratch bytes qgemm_quantize_act / qgemm_quantize_weight need (NVFP4 keeps
 * its per-CTA amax partials there; the 8-bit formats need none: 0). */
size_t qgemm_quant_workspace_size(qg_format f, int rows, int K);

/* Scratch bytes qgemm_run needs for this configuration: 0 when split_k == 1
 * or reduce_mode == 0; split_k * M * N * 4 bytes of partial sums (rounded up
 * to 256) for reduce_mode 1; the same plus one 4-byte arrival counter per
 * output tile for reduce_mode 2.  The counter region must be zero before the
 * first reduce_mode-2 call (see qgemm_workspace_clear); every completed call
 * leaves it zero again. */
size_t qgemm_workspace_size(qg_format f, int M, int N, int K, const qg_config* cfg);

/* Zeroes a run workspace on `stream` (one cudaMemsetAsync). */
qg_status qgemm_workspace_clear(void* workspace, size_t ws_bytes, void* stream);

/* ----------------------------------------------------------- quantisers -- */

/* Dynamic activation quantisation (the "quantization" auxiliary kernel of
 * "Helion in the vLLM backend", seventh paragraph), fused in one pass per
 * row / group: amax over the row (FP8_DYNAMIC, W8A8_INT8), the 1x128 group
 * (BLOCK_FP8) or the tensor and each 16-element block (NVFP4), then
 * scale = amax / Qmax (448 for e4m3, 127 for int8) in correctly rounded fp32,
 * and codes = round-to-nearest-even(x / scale) saturated to the format
 * (int8 clamped to [-127, 127]).  An all-zero row/group/tensor gets scale 1.
 * NVFP4: g = amax(tensor) / 2688, block scale = e4m3((amax_b / 6) / g),
 * code = e2m1(x / (dec(block scale) * g)), code 0 where the block scale is 0.
 *
 *   A:   bf16 [M, lda] (lda >= K elements, lda*2 a multiple of 16 bytes)
 *   static_amax: NVFP4 only, optional device fp32 scalar; when non-NULL it
 *        replaces the tensor amax (a static activation scale).
 *   out: caller-allocated q / scale / global_scale of the sizes
 *        qgemm_operand_bytes(f, 0, M, K) gives; out->rows = M, out->K = K.
 *   workspace: qgemm_quant_workspace_size(f, M, K) bytes (NULL if 0).
 * K must be a multiple of 16 (FP8_DYNAMIC, W8A8_INT8), 128 (BLOCK_FP8) or
 * 32 (NVFP4). */
qg_status qgemm_quantize_act(qg_format f, const void* A, int M, int K, int lda,
                             const float* static_amax, qg_operand* out,
                             void* workspace, size_t ws_bytes, void* stream);

/* Offline weight quantisation of W bf16 [N, K] (contiguous): per-channel
 * (FP8_DYNAMIC: amax/448, W8A8_INT8: amax/127), per 128x128 block
 * (BLOCK_FP8) or NVFP4 as above. */
qg_status qgemm_quantize_weight(qg_format f, const void* W, int N, int K, qg_operand* out,
                                void* workspace, size_t ws_bytes, void* stream);

/* Mixture-of-experts operands for qgemm_run_grouped.
 *
 * qgemm_grouped_act_bytes: the `q` and `scale` bytes of the activation
 * operand of T tokens routed over `experts` experts: those of
 * qgemm_operand_bytes(f, 0, T, K) except NVFP4, whose block scales take
 * floor((T - a) / 128) + a 128-row atoms, a = min(experts, T) (every active
 * expert may open a fresh atom).
 *
 * qgemm_quantize_act_grouped: qgemm_quantize_act of bf16 A [T, lda], tokens
 * sorted by expert, expert e owning rows [expert_offsets[e],
 * expert_offsets[e + 1]) (DEVICE int32 [experts + 1], read after the wait on
 * the preceding kernel, clamped to [0, T]).  The 8-bit formats' scales are
 * per token or token group, so this is qgemm_quantize_act.  NVFP4: one
 * tensor scale over all T tokens (the activation is one tensor), codes
 * [T, K/2] as usual, and block scales in the per-expert layout: expert e's
 * scale rows start at 128 x sum_{e' < e} ceil(c_e' / 128) (c the token
 * counts), its tokens in order, the rest of its last atom zero, so each
 * expert's scales are the plain 128x4 tiled layout of its own c_e rows.
 * out->scale holds qgemm_grouped_act_bytes bytes; out->rows = T.
 *
 * qgemm_quantize_weight_grouped: qgemm_quantize_weight of the stacked
 * weights W bf16 [experts * N, K], N a multiple of 128; out->rows =
 * experts * N.  The 8-bit formats' per-channel and 128x128-block scales
 * never cross an expert, so this is qgemm_quantize_weight of the stack.
 * NVFP4: every expert is quantised as its own tensor (its own tensor scale,
 * out->global_scale [experts]); its codes and block scales sit at
 * e x qgemm_operand_bytes(f, 1, N, K) in the stacked buffers.  workspace:
 * qgemm_quant_workspace_size(f, N, K) bytes, reused by each expert in turn.
 * experts: 1 ... 256. */
qg_status qgemm_grouped_act_bytes(qg_format f, int experts, int T, int K, size_t* q_bytes,
                                  size_t* scale_bytes);
qg_status qgemm_quantize_act_grouped(qg_format f, int experts, const int* expert_offsets, const void* A,
                                     int T, int K, int lda, const float* static_amax, qg_operand* out,
                                     void* workspace, size_t ws_bytes, void* stream);
qg_status qgemm_quantize_weight_grouped(qg_format f, int experts, const void* W, int N, int K,
                                        qg_operand* out, void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ GEMM -- */

/* y = dequant(A_q) . dequant(W_q)^T with configuration `cfg`.
 *   A: activations, A->rows == M, A->K == K;  W: weights, W->rows == N.
 *   Y: bf16 [M, ldy] (QG_OUT_BF16) or int32/fp32 [M, ldy] (QG_OUT_ACC);
 *      ldy >= N, ldy * elem a multiple of 16 bytes.
 *   workspace: qgemm_workspace_size(f, M, N, K, cfg) bytes (NULL if 0).
 * Epilogue: y = acc * s_a[m] * s_w[n] (FP8_DYNAMIC, W8A8_INT8; int32 acc
 * converted to fp32 first), per-group promotion acc += p_g
 * (s_a[m,g] * s_w[n/128,g]) as one fp32 FMA per element (BLOCK_FP8),
 * y = acc * (g_a * g_w) (NVFP4); all in fp32, then
 * bf16 round-to-nearest-even.  Returns QG_ERR_UNSUPPORTED for a config the
 * kernels do not implement (e.g. split_k larger than the number of 128-byte
 * K tiles) and QG_ERR_WORKSPACE if ws_bytes is too small.
 * Weights are read before the kernel waits on the preceding kernel of the
 * stream (programmatic dependent launch): W_q must not be written by a
 * kernel that may still run when qgemm_run is enqueued. */
qg_status qgemm_run(qg_format f, const qg_operand* A, const qg_operand* W, int M, int N, int K,
                    const qg_config* cfg, void* workspace, size_t ws_bytes, void* Y, int ldy,
                    int out_kind, void* stream);

/* Grouped GEMM for a mixture-of-experts layer ("Helion in the vLLM
 * backend", last paragraph: an MoE backend is the next target): for every
 * expert e and every token t routed to it,
 *     y[t, :] = dequant(A_q)[t, :] . dequant(W_q[e])^T,
 * in one launch.  Tokens are sorted by expert: expert e owns rows
 * [expert_offsets[e], expert_offsets[e + 1]) of A and y.
 *   experts:        1 ... 256.
 *   expert_offsets: DEVICE int32 [experts + 1], nondecreasing, [0] = 0,
 *                   [experts] = A->rows; read by the kernel after it waits on
 *                   the preceding kernel of the stream (the routing), so the
 *                   call needs no host copy and can be captured.  Offsets
 *                   outside [0, A->rows] are clamped on the device.
 *   A:  activations of all T = A->rows tokens (quantised as one operand,
 *       by qgemm_quantize_act_grouped with the same offsets: for NVFP4 its
 *       block scales are in the per-expert layout that call documents).
 *   W:  all experts' weights stacked, W->rows = experts * N, expert e's rows
 *       at [e * N, (e + 1) * N); per-channel scales [experts * N] or 128x128
 *       block scales [experts * N / 128, K / 128]; NVFP4: block scales of
 *       the stacked rows and one tensor scale per expert, global_scale
 *       [experts] (qgemm_quantize_weight_grouped).  N must be a multiple of
 *       128 (no 128-row block straddles two experts).
 *   Y:  [T, ldy]; cfg: swap_ab = 1 (a decode expert sees few tokens), any
 *       split_k with reduce_mode 0 or 1 (workspace as qgemm_workspace_size(f,
 *       T, N, K, cfg)); tile_n is the token tile.
 * The grid covers floor((T - a) / tile_n) + a token tiles, a = min(experts,
 * T): the most that any routing of T tokens over the experts needs.  A CTA
 * finds its expert and tokens with a warp scan over the offsets and exits if
 * it has none.  Weights are loaded after that lookup (which experts run depends on
 * the routing).  All four formats; NVFP4 takes tile_n >= 64 unless T <=
 * tile_n (a token tile's block scales must start at an even 32-row word of
 * its expert's 128-row scale atom). */
qg_status qgemm_run_grouped(qg_format f, int experts, const int* expert_offsets, const qg_operand* A,
                            const qg_operand* W, int N, int K, const qg_config* cfg, void* workspace,
                            size_t ws_bytes, void* Y, int ldy, int out_kind, void* stream);

/* Default configuration of a grouped launch of T tokens over `experts`
 * experts, without the routing: at most min(experts, T) experts are active
 * and the launch streams their weights, so the configuration is the
 * scorer's first-ranked one for min(experts, T) * N weight rows and
 * ceil(T / active) tokens among those qgemm_run_grouped accepts (swap_ab = 1,
 * reduce_mode 0 or 1); else split_k 1, tile_n 16 (NVFP4 with T > 16: 64),
 * 4 stages. */
qg_status qgemm_grouped_default_config(qg_format f, int experts, int T, int N, int K, qg_config* out);

/* Activation quantisation fused into the GEMM: y = dequant(quant(A)) .
 * dequant(W_q)^T for bf16 activations A, in one kernel.  The pages name the
 * dynamic activation quantisation among the auxiliary kernels around the
 * linear-layer GEMM ("Helion in the vLLM backend", seventh paragraph); here
 * the GEMM's epilogue warps, idle during the mainloop, quantise the
 * activation slice of their CTA into the shared-memory ring themselves, so a
 * decode step makes one launch instead of two and the quantised activations
 * never go through HBM.  The codes and scales are those qgemm_quantize_act
 * computes (same arithmetic, bit for bit), so y is bitwise equal to
 * qgemm_quantize_act followed by qgemm_run with the same configuration.
 *   A:   bf16 [M, lda], 16-byte aligned, lda >= K, lda*2 a multiple of 16.
 *   W, M, N, K, cfg, workspace, Y, ldy, out_kind: as for qgemm_run.
 *   act_scale_out: optional fp32 output of the activation scales the kernel
 *        used: [M] (FP8_DYNAMIC, W8A8_INT8) or [M, K/128] (BLOCK_FP8).
 * Supported: FP8_DYNAMIC, W8A8_INT8 and BLOCK_FP8 with swap_ab = 1 (the
 * decode orientation).  A per-token scale spans all of K, so FP8_DYNAMIC and
 * W8A8_INT8 need split_k = 1 or reduce_mode 0 (the split-K CTAs of a tile
 * form a cluster and exchange partial amaxes through distributed shared
 * memory); BLOCK_FP8 groups are local to a K tile and take any split.
 * NVFP4 (whose tensor scale needs the amax of all of A) and swap_ab = 0
 * return QG_ERR_UNSUPPORTED; bad pointers, strides or sizes
 * QG_ERR_INVALID_ARG; all checks happen on the host before any launch.
 * The caller owns every buffer; nothing is allocated. */
qg_status qgemm_run_fused_act(qg_format f, const void* A, int lda, const qg_operand* W, int M, int N,
                              int K, const qg_config* cfg, void* workspace, size_t ws_bytes, void* Y,
                              int ldy, int out_kind, float* act_scale_out, void* stream);

/* qgemm_run without a caller-provided workspace.  There is no counterpart of
 * this entry point in the pages the library follows; it exists for callers
 * that cannot allocate device memory on this path (an engine whose memory
 * planner reserved all device memory up front and forbids allocation while
 * serving, a plugin host that passes only input and output buffers).  Inputs
 * and outputs are still the caller's; the split-K scratch (reduce_mode 1 or
 * 2) comes from a fixed array inside the library, QGEMM_NOALLOC_SCRATCH_BYTES
 * bytes on every GPU that loads the library, held until the process exits.
 *   - A configuration whose qgemm_workspace_size exceeds that maximum is
 *     rejected with QG_ERR_WORKSPACE before any device work.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.  A first call on a device made while
 *     `stream` is being captured is refused with QG_ERR_UNSUPPORTED.
 *   - No cudaMalloc, cudaFree or other allocation is made.  For reduce_mode 2
 *     the tile-counter region is cleared with cudaMemsetAsync on `stream`.
 *   - Every call shares the one array and it keeps the last call's contents:
 *     calls that overlap on the GPU (other streams, other threads) race on it
 *     and must be serialised by the caller.
 * Other arguments and results are those of qgemm_run. */
#define QGEMM_NOALLOC_SCRATCH_BYTES (8u << 20)
qg_status qgemm_run_noalloc(qg_format f, const qg_operand* A, const qg_operand* W, int M, int N,
                            int K, const qg_config* cfg, void* Y, int ldy, int out_kind,
                            void* stream);

/* Default configuration for a shape when no table entry exists: the
 * configuration qgemm_rank_configs ranks first (the zero-tune default of
 * FlashInfer PR 3948's tactic heuristic).  If no candidate of the scorer's
 * grid is feasible, a fixed rule: swap_ab = 1 up to 64 tokens ("Helion in
 * the vLLM backend", second paragraph: vLLM's Block_FP8 backend swaps A and
 * B below M = 32), split_k chosen so that output tiles x split_k approaches
 * the SM count, the deepest ring that fits. */
qg_status qgemm_default_config(qg_format f, int M, int N, int K, qg_config* out);

/* Analytic tactic scorer (FlashInfer PR 3948: rank tactics with a heuristic
 * from the shape -- wave quantisation, efficiency, feasibility -- and tune
 * only the top N).  The model estimates a launch's time from the bytes each
 * CTA streams through its ring (Little's law: in-flight bytes / latency, per-SM
 * and HBM caps), the MMA loop's cycles per K tile (plus Block_FP8
 * promotion), waves over the SMs (shared memory, registers and TMEM columns
 * per CTA) and the split-K reduction of each mode; its constants were fitted
 * to the tuner's measurements of every candidate on one B200.  Host only, no
 * device work, capture-safe.
 *   qgemm_score_config: *est_us = the estimate for one configuration;
 *     returns the qgemm_run status of the configuration if it is invalid.
 *   qgemm_rank_configs: the feasible configurations of the tuner's candidate
 *     grid, best estimate first, written to out[0 .. *n_out) (at most
 *     max_out; est_us, if not NULL, receives the estimates).  Deterministic. */
qg_status qgemm_score_config(qg_format f, int M, int N, int K, const qg_config* cfg, double* est_us);
qg_status qgemm_rank_configs(qg_format f, int M, int N, int K, qg_config* out, int max_out, double* est_us,
                             int* n_out);

/* ---------------------------------------------------- table and tuning -- */

/* Loads a per-shape table file written by qgemm_tune / qgemm_table_save.
 * *table receives a library-owned handle, freed by qgemm_table_free. */
qg_status qgemm_table_load(const char* path, void** table);
/* Creates an empty table. */
qg_status qgemm_table_create(void** table);
/* Inserts or replaces the entry for (f, M, N, K). */
qg_status qgemm_table_put(void* table, qg_format f, int M, int N, int K, const qg_config* cfg,
                          double us);
/* Writes the table (text, versioned, with device name and SM count). */
qg_status qgemm_table_save(const void* table, const char* path);
void qgemm_table_free(void* table);
/* Number of entries. */
int qgemm_table_size(const void* table);

/* Looks up (f, M, N, K).  *hit = 1 on an exact entry.  On a miss the entry
 * with the same (f, N, K) and the smallest tuned M' >= M is used (*hit = 2):
 * tuned token counts act as buckets -- decode (M <= 32), medium (64 ... 2048)
 * and large -- as in TensorRT-LLM issue 16363's policy buckets.  Failing
 * that, qgemm_default_config (*hit = 0).  Identity gate: a table whose
 * recorded device name or SM count differs from the current device's is not
 * used at all (*hit = -1, qgemm_default_config); without a device, or for a
 * table that records none ("unknown" / 0 SMs), no gate applies.  Host only,
 * no device work beyond reading the device's properties, capture-safe. */
qg_status qgemm_dispatch(const void* table, qg_format f, int M, int N, int K, qg_config* out,
                         int* hit);

/* Ahead-of-time tuner: for each (M, (N, K)) enumerates the valid configs
 * (split_k, swap_ab, tile_n, stages, reduce_mode), times each with CUDA
 * events over a graph of back-to-back layer steps -- qgemm_quantize_act then
 * qgemm_run, as a layer with dynamic activations runs them (selection pass),
 * re-times the winner in an independent pass whose step time is what the
 * table records, and rejects any config whose output differs from the
 * default config's.  Among configs within 10% of the fastest it picks one
 * whose ring holds every K tile of its split (all weights requested before
 * the dependency wait), which keeps its time next to kernels of other shapes
 * and after graph boundaries, where the same-shape timing loop is blind.
 * Shapes already
 * present in `table` are skipped (resume).  Synthetic inputs are generated
 * on the device; `budget_s_per_shape` bounds the wall time per shape.
 * NK holds nNK pairs (N, K). */
qg_status qgemm_tune(void* table, qg_format f, const int* Ms, int nM, const int* NK, int nNK,
                     double budget_s_per_shape, int verbose);
/* Validation gate of a table (TensorRT-LLM issue 16363's shape-gated policy:
 * a configuration that fails validation falls back to a known-good one).
 * Runs every entry on synthetic inputs of its shape next to the scored
 * default configuration (qgemm_default_config) and removes the entries that
 * the kernels refuse on this device or whose bf16 output leaves
 * |y - y_default| <= 0.01 |y_default| + 0.01 rms(y_default row); dispatch
 * then answers those shapes with the default.  *checked / *rejected receive
 * the counts.  Allocates device memory and synchronises: an offline step (at
 * table load), not a run-path call.  verbose != 0 prints each rejection. */
qg_status qgemm_table_validate(void* table, int* checked, int* rejected, int verbose);

/* qgemm_tune over the top_n configurations qgemm_rank_configs ranks first
 * instead of the whole grid (top-N pruned tuning, FlashInfer PR 3948's
 * "autotune over a top-N ranked list"); the other arguments and the table
 * entries are those of qgemm_tune. */
qg_status qgemm_tune_ranked(void* table, qg_format f, const int* Ms, int nM, const int* NK, int nNK,
                            int top_n, double budget_s_per_shape, int verbose);
/* Tuning instrumentation: while `path` is set (NULL clears it), qgemm_tune
 * appends one text line per timed candidate to that file:
 *   <fmt> <M> <N> <K> <split_k> <swap_ab> <tile_n> <stages> <reduce_mode> <variant> <rows> <us>
 * (the selection-pass step time).  Host only; not thread-safe. */
void qgemm_set_tune_log(const char* path);

/* What the tuner times per candidate: gemm_only = 0 (the default) replays
 * steps of a linear layer, the dynamic activation quantisation followed by
 * the GEMM (their overlap through programmatic dependent launch depends on
 * the configuration); gemm_only = 1 replays back-to-back GEMMs alone, the
 * per-shape time of the GEMM itself.  Host only; not thread-safe. */
void qgemm_set_tune_objective(int gemm_only);

/* -------------------------------------------------------------- errors -- */

const char* qgemm_status_string(qg_status s);
/* Reads (and clears) the device error word set by a bounded in-kernel wait
 * that expired; synchronises the device.  Returns QG_OK or
 * QG_ERR_DEVICE_TIMEOUT. */
qg_status qgemm_device_error(void);

/* Limit of every bounded in-kernel wait of later launches, in ns of the GPU's
 * %globaltimer (0 restores the default of 200 ms).  On expiry a wait sets the
 * device error word (QG_ERR_DEVICE_TIMEOUT from qgemm_device_error) and the
 * kernel leaves its loops, waits (bounded) for its own copies in flight,
 * frees its TMEM and returns, so the context stays usable.  Host state, not
 * thread-safe. */
void qgemm_set_wait_limit(unsigned long long limit_ns);

/* Failure-detection self-test: launches one CTA on `stream` that waits, with
 * the library's bounded wait and a limit of `limit_ns` (1 ns .. 200 ms), on
 * an mbarrier nothing arrives on.  The wait expires and sets the device error
 * word, which the next qgemm_device_error reports (QG_ERR_DEVICE_TIMEOUT) and
 * clears.  No copy or MMA is in flight, so the kernel returns normally.
 * QG_ERR_INVALID_ARG for a limit outside that range; QG_ERR_CUDA if the
 * launch fails. */
qg_status qgemm_selftest_wait_expiry(unsigned long long limit_ns, void* stream);
/* Enables (1) or disables (0) programmatic dependent launch for the
 * library's kernels (default 1). */
void qgemm_set_pdl(int enable);
/* Enables (1) or disables (0) TMA stores of the output tile (default 1):
 * launches in the standard orientation (swap_ab = 0) with split_k = 1,
 * tile_n >= 64 and bf16 output write their tile through a tensor map of y
 * instead of thread stores (same values, bit for bit).  A switch for
 * comparison and tests. */
void qgemm_set_tma_store(int enable);
/* Tracing (debug): while set, every qgemm_run whose grid fits records, per
 * CTA, 15 GPU-clock timestamps (%globaltimer, ns, 64-bit) into the device
 * buffer: entry, set-up done, first weight tile issued, dependency wait
 * returned, first stage landed, last MMA committed, accumulator ready, stores
 * done, and for cluster split-K: partial pushed, owned slices received,
 * owned rows reduced; word 11: the MMA issuer saw the last full stage.  In a
 * fused launch (qgemm_run_fused_act) word 3 is the epilogue warps' dependency
 * wait and words 12-14 mark the activation slice's local maxima, the
 * cluster's exchanged maxima and the published codes.  Words not reached
 * stay as they were.  CTA c = (z * gridDim.y + y) * gridDim.x + x writes
 * words [15c, 15c+15).
 * Launches whose grid needs more than `bytes` are not traced.  NULL turns
 * tracing off.  Not thread-safe; meant for profiling runs. */
void qgemm_set_trace(void* device_buffer, size_t bytes);

/* ABI version of the loaded library (QGEMM_ABI_VERSION). */
int qgemm_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* QGEMM_H_ */
