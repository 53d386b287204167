// gemm_kernel.cuh — the unified quantized GEMM kernel for sm_100a.
//
// One CTA computes an output tile D[128 x BN] over a slice of the K tiles:
//   D[p, q] = sum_k P[p, k] * Q[q, k]
// P is the 128-row MMA operand and Q the BN-row one, both K-contiguous.
// Standard orientation: P = A_q (tokens), Q = W_q (channels).
// Swap-AB ("Helion in the vLLM backend", second paragraph: A@B rewritten as
// (B^T A^T)^T): P = W_q, Q = A_q, so the weight rows fill the 128-row MMA
// slot and a handful of tokens fill N = 16 or 32.
//
// Warp roles (64 threads + the epilogue warps):
//   warp 0      TMA producer: weights first (they do not depend on the
//               preceding kernel), then griddepcontrol.wait, then activations;
//               a `stages`-deep ring of 128-byte K tiles in shared memory.
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer.
//   warps 2..   epilogue, 4 warps (Block_FP8 with 128- or 256-wide tiles: 8
//               or 16): tcgen05.ld of the fp32/int32 accumulator, scales in
//               fp32, bf16 store, or this CTA's split-K partial.
// Block_FP8 promotes every 128-wide K group: the MMA writes the group's
// partial sum into one of NACC TMEM buffers and the epilogue warps fold it
// into fp32 registers with the group's activation and weight-block scales.
// NVFP4 uses kind::mxf4nvf4 with the e4m3 block scales copied
// smem -> TMEM by tcgen05.cp.
//
// Split-K ("Helion in the vLLM backend", second and third paragraphs): the
// split_k CTAs of one output tile either form a thread-block cluster and
// meet in distributed shared memory (no global scratch), or leave partials
// in a workspace that the last-arriving CTA or a second kernel sums.  In the
// cluster, narrow tiles push each row's partial to the CTA that owns it with
// asynchronous stores that count their bytes on the owner's barrier; the
// owner sums and stores units of 8 channels in one pass.  Wide tiles stage
// their partial in the idle ring and the owners pull.  Every mode adds the
// partials in split order, so results are deterministic and identical
// across modes.
//
// Grouped (mixture-of-experts) launches read device-side expert offsets after
// the dependency wait; each CTA finds its expert and token tile with a warp
// scan, and CTAs without a tile leave before any set-up.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "ptx.cuh"
#include "quant_math.cuh"

namespace qg {

enum Fmt : int { kFP8 = 0, kINT8 = 1, kBLOCK = 2, kNVF4 = 3 };

constexpr int kKTileBytes = 128;     // bytes of K per pipeline stage (one 128B swizzle row)
constexpr int kPTileBytes = 128 * kKTileBytes;
constexpr int kSfAtomBytes = 512;    // one 128x4 atom of e4m3 block scales

constexpr int kReduceCluster = 0;    // split-K partials summed through distributed shared memory
constexpr int kReduceSecondPass = 1; // partials in the workspace, summed by a second kernel
constexpr int kReduceLastCta = 2;    // partials in the workspace, summed by the last-arriving CTA
constexpr int kMaxClusterSplit = 8;

// How the activation (Q) tiles of a Swap-AB launch reach shared memory.
// TMA: the quantised codes stream through the ring, one box per stage next to
// the weight tile.  Fused: the epilogue warps (idle until the accumulator is
// ready) quantise this CTA's bf16 activation slice, K tiles [kt_begin,
// kt_end), into a dedicated region once and publish it through one barrier;
// the ring then carries only weights.
constexpr int kActTma = 0;
constexpr int kActFused = 1;

struct GemmParams {
  int M, N, K;
  int rows_p, rows_q;          // rows of the P / Q operands
  int kt_total;                // 128-byte K tiles
  int split_k;
  int stages;
  int groups;                  // Block_FP8: K / 128
  const float* scale_a;        // activation scales (per token, or [M, groups])
  const float* scale_w;        // weight scales (per channel, or [ceil(N/128), groups])
  const uint8_t* sf_p;         // NVFP4 block scales of P / Q (128x4 layout)
  const uint8_t* sf_q;
  int sf_atoms_per_rb;         // NVFP4: 128x4 atoms per 128-row block (= ceil(K/256)*4)
  const float* g_a;            // NVFP4 tensor scales
  const float* g_w;
  void* Y;
  int ldy;
  int out_kind;                // 0 = bf16, 1 = raw accumulators
  void* partial;               // split-K partials [split][M][N] (4-byte elements)
  unsigned int* counters;      // split-K per-tile arrival counters
  int reduce_mode;             // kReduce*
  unsigned int* err;           // device error word
  unsigned long long wait_ns;  // limit of every in-kernel wait (ns)
  unsigned long long* trace;   // optional: kTraceEvents timestamps per CTA (ns)
  int nkt_max;                 // most K tiles any split slice holds: ceil(kt_total / split_k)
  int recv_cols;               // cluster push: token columns per receive slot (0: no receive buffer)
  // Fused activation quantisation (Swap-AB; FP8_Dynamic, W8A8_INT8,
  // Block_FP8): with `act` set, the epilogue warps read the bf16 activations,
  // quantise them exactly as the standalone quantiser does and write the
  // codes into the ring's Q tiles; `act` null selects the TMA-fed A_q path.
  const __nv_bfloat16* act;    // bf16 A [M, lda]
  int lda;
  float* act_scale_out;        // optional: the activation scales (per token, or [M, K/128])
  int a_mode;                  // kActTma / kActFused: how the Q (activation) tiles fill
  // Grouped (mixture-of-experts) launch: tokens sorted by expert, expert e
  // owning rows [expert_offsets[e], expert_offsets[e + 1]) of A and y, and
  // weight rows [e * N, (e + 1) * N) of W_q.
  const int* expert_offsets;   // device, experts + 1 ints
  int experts;
  // Weight prefetch into L2 on behalf of a later CTA: the CTA `l2_ahead`
  // places after this one in launch order (same split slice in a cluster
  // launch), 0 for none.  CTAs that start while the previous kernel still
  // holds the SMs stream the weights of those that can only start after it,
  // so the HBM stays busy across the kernel boundary.
  int l2_ahead;
  // Standard orientation, no split, bf16 out, BN >= 64: the epilogue writes
  // the bf16 tile into the idle ring in boxes of 128 rows x 64 channels with
  // the 128-byte swizzle and stores them with TMA through the y tensor map
  // (kernel parameter); 0: 16-byte stores from the threads.
  int y_tma;
};

constexpr int kMaxExperts = 256;

// Phase timestamps (%globaltimer, ns) a traced launch records per CTA.
enum TraceEvent : int {
  kTrEntry = 0,        // kernel entry
  kTrReady = 1,        // barriers initialised, TMEM allocated
  kTrFirstLoad = 2,    // producer issued its first weight tile
  kTrDepWait = 3,      // producer returned from griddepcontrol.wait
  kTrFirstFull = 4,    // MMA issuer saw the first full stage
  kTrLastMma = 5,      // MMA issuer committed its last MMA
  kTrAccReady = 6,     // epilogue has the (promoted) accumulator
  kTrDone = 7,         // epilogue finished its stores
  kTrSent = 8,         // cluster split-K: partial rows pushed to their owners
  kTrRecv = 9,         // cluster split-K: owned slices received
  kTrReduced = 10,     // cluster split-K: owned rows summed into the output tile
  kTrLastFull = 11,    // MMA issuer saw the last full stage
  kTrActLoaded = 12,   // fused: the slice's per-token maxima of this CTA are known
  kTrActAmax = 13,     // fused: the cluster's maxima exchanged (the scales are known)
  kTrActReady = 14,    // fused: the codes are published to the tensor core
  kTraceEvents = 15
};
__device__ __forceinline__ void trace_at(const GemmParams& prm, int ev) {
  if (prm.trace != nullptr) {
    const size_t cta = ((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
    prm.trace[cta * kTraceEvents + ev] = globaltimer();
  }
}

template <int FMT, int BN>
struct Cfg {
  static constexpr bool kBlock = FMT == kBLOCK;
  static constexpr bool kNvf4 = FMT == kNVF4;
  static constexpr bool kRowColScales = FMT == kFP8 || FMT == kINT8;
  static constexpr int kQTileBytes = BN * kKTileBytes;
  static constexpr int kSfQAtoms = BN > 128 ? 2 : 1;               // 128-row SF blocks of Q
  static constexpr int kSfPBytes = kNvf4 ? 4 * kSfAtomBytes : 0;   // 4 K-atoms per 128B tile
  static constexpr int kSfQBytes = kNvf4 ? 4 * kSfAtomBytes * kSfQAtoms : 0;
  static constexpr int kNAcc = kBlock ? (BN >= 256 ? 2 : 4) : 1;  // Block_FP8 group buffers
  // Wide Block_FP8 tiles promote with more epilogue warps: two (BN = 128) or
  // four (BN = 256) per 32-lane TMEM quarter, each owning a share of the
  // columns, so that while some warps wait on their TMEM loads others run
  // their FMAs (a warp's promotion is a chain of load -> wait -> FMA).
  static constexpr int kEpiWarps = (kBlock && BN >= 256) ? 16 : (kBlock && BN >= 128) ? 8 : 4;
  static constexpr int kEpiThreads = 32 * kEpiWarps;
  static constexpr int kThreads = 64 + kEpiThreads;
  static constexpr int kCols = BN / (kEpiWarps / 4);               // columns per epilogue thread
  // CTAs per SM the register budget must allow: narrow (decode) tiles keep
  // room for the next launch's CTAs to start streaming weights early.
  static constexpr int kMinBlocks = (!kBlock && BN <= 64) ? 3 : (kBlock && BN <= 32) ? 2 : 1;
  static constexpr int kAccCols = kNAcc * BN;                      // accumulator columns
  static constexpr int kSfaCol = kAccCols;                         // TMEM column of SF A
  static constexpr int kSfbCol = kSfaCol + 16;                     // 4 steps x 4 words
  static constexpr int kTmemUsed = kNvf4 ? kSfbCol + 16 * kSfQAtoms : kAccCols;
  static constexpr int kTmemCols = kTmemUsed <= 32    ? 32
                                   : kTmemUsed <= 64  ? 64
                                   : kTmemUsed <= 128 ? 128
                                   : kTmemUsed <= 256 ? 256
                                                      : 512;
  static constexpr uint32_t kIdesc = kNvf4              ? idesc_nvf4(BN)
                                     : (FMT == kINT8)   ? idesc_i8(BN)
                                                        : idesc_f8f6f4_e4m3(BN);
  // Cluster split-K for narrow tiles pushes partial slices into a dedicated
  // receive buffer of the owning CTA; wide tiles pull from the ring instead.
  static constexpr bool kPush = BN <= 64;
};

// Two MMA-issuing threads (Swap-AB FP8_Dynamic / W8A8_INT8 whose ring holds
// every K tile of the slice): the MMA warp issues the even K tiles into one
// accumulator and the producer thread, idle once its loads are out, the odd
// ones into a second; the epilogue adds the two.  At decode sizes one
// thread's issue of four small MMAs and a commit per K tile is on the
// critical path, and two threads issue in parallel.  The plain, fused and
// grouped launches split the same way, so that for one configuration they
// sum in the same order.
template <int FMT, bool SWAP, int BN, bool FUSED, bool GROUPED>
__host__ __device__ constexpr bool dual_issue_able() {
  return SWAP && (FMT == kFP8 || FMT == kINT8);
}
template <int FMT, bool SWAP, int BN, bool FUSED, bool GROUPED>
__host__ __device__ constexpr int tmem_cols() {
  using C = Cfg<FMT, BN>;
  if constexpr (dual_issue_able<FMT, SWAP, BN, FUSED, GROUPED>()) {
    return 2 * C::kAccCols <= 32 ? 32 : 2 * C::kAccCols <= 64 ? 64 : 2 * C::kAccCols <= 128 ? 128
           : 2 * C::kAccCols <= 256 ? 256 : 512;
  } else {
    return C::kTmemCols;
  }
}

// Block_FP8 scales staged per CTA: activation rows x K tiles, then weight
// blocks x K tiles.
template <bool SWAP, int BN>
__host__ __device__ constexpr int block_act_rows() { return SWAP ? BN : 128; }
template <bool SWAP, int BN>
__host__ __device__ constexpr int block_weight_blocks() { return (!SWAP && BN > 128) ? 2 : 1; }

// Shared-memory carve-up (offsets from a 1024-byte aligned base).  The
// receive buffer and the Block_FP8 scale area are sized by the launch (its
// token count and K slice), so decode launches stay small enough for several
// CTAs per SM: the next launch's CTAs then stream weights while this one ends.
struct SmemLayout {
  uint32_t p, q, sfp, sfq, recv, bars, misc, epis, scales, fuse, total;
};
// Fused activation prologue: this CTA's per-token amax, then one slot of
// partial amaxes per split-K peer of the cluster.
template <int FMT, bool SWAP, int BN>
__host__ __device__ constexpr uint32_t fuse_bytes() {
  return (SWAP && FMT != kNVF4) ? 4u * (uint32_t)((1 + kMaxClusterSplit) * BN) : 0u;
}
template <int FMT, bool SWAP, int BN>
__host__ __device__ inline SmemLayout smem_layout(int stages, int nkt_max, int recv_cols, int act_tiles) {
  using C = Cfg<FMT, BN>;
  SmemLayout L;
  L.p = 0;
  L.q = L.p + stages * kPTileBytes;
  // Q tiles: one per stage in the ring, or (act_tiles > 0) the activation
  // slice of the whole K range, one tile per K tile
  L.sfp = L.q + (act_tiles > 0 ? act_tiles : stages) * C::kQTileBytes;
  L.sfq = L.sfp + stages * C::kSfPBytes;
  L.recv = L.sfq + stages * C::kSfQBytes;
  L.bars = L.recv + (C::kPush ? 4u * 128u * (uint32_t)recv_cols : 0u);
  // full[stages], empty[stages], acc_full, tfull[4], tempty[4], recv_full, amax_full, act_ready
  L.misc = L.bars + 8 * (2 * stages + 1 + 8 + 3);
  L.epis = (L.misc + 16 + 15) & ~15u;          // row / column scales (FP8, INT8)
  L.scales = L.epis + (C::kRowColScales ? 4 * (128 + BN) : 0);
  L.fuse = L.scales + (C::kBlock ? 4u * (uint32_t)((block_act_rows<SWAP, BN>() +
                                                    block_weight_blocks<SWAP, BN>()) * nkt_max)
                                 : 0u);
  L.total = L.fuse + fuse_bytes<FMT, SWAP, BN>();
  return L;
}
template <int FMT, bool SWAP, int BN>
__host__ inline size_t smem_bytes(int stages, int nkt_max, int recv_cols, int act_tiles) {
  return smem_layout<FMT, SWAP, BN>(stages, nkt_max, recv_cols, act_tiles).total + 1024;  // + alignment slack
}

// Bytes a pull-mode cluster reduction stages in the (then idle) ring.
template <bool SWAP, int BN>
__host__ __device__ constexpr int red_bytes() {
  return SWAP ? 4 * 128 * BN : 4 * 128 * (BN + 4);
}
// Position of accumulator element (row of P, column c) in the pull-mode
// buffer: the output-tile layout (channels contiguous, 16-byte aligned
// groups of 8 along them).
template <bool SWAP, int BN>
__device__ __forceinline__ int red_index(int row, int c) {
  return SWAP ? c * 128 + row : row * (BN + 4) + c;
}
// Output tile: element (row r of P, column c) of the raw accumulator tile.
// Swap-AB keeps channels (r) contiguous, the standard orientation keeps
// channels (c) contiguous with a padded row pitch; both are 16-byte aligned
// for every 8-element group along the contiguous dimension.
template <bool SWAP, int BN>
__device__ __forceinline__ int tile_index(int r, int c) {
  return SWAP ? c * 128 + r : r * (BN + 4) + c;
}
template <bool SWAP, int BN>
__host__ __device__ constexpr int tile_bytes() {
  return SWAP ? 4 * 128 * BN : 4 * 128 * (BN + 4);
}
// Push mode (standard orientation): CTA `owner` receives rows [owner*rows_per, (owner+1)*rows_per)
// of every split's partial; slot z holds split z's slice, laid out so the
// owner's final stores are coalesced.
template <bool SWAP, int BN>
__device__ __forceinline__ int slice_index(int rl, int c, int rows_per) {
  return SWAP ? c * rows_per + rl : rl * BN + c;
}

__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// Named barrier over n threads that returns to every one of them whether
// any passed `v` true: a decision all of them take the same way (a flag
// another role may set meanwhile, read once per thread, would not be).
__device__ __forceinline__ bool named_bar_or(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, %3, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ uint32_t ld_u32_cg(const void* p) {
  return __ldcg(reinterpret_cast<const unsigned int*>(p));
}

// Epilogue scale of one output element, before bf16 rounding.
template <int FMT>
__device__ __forceinline__ float finish_value(uint32_t acc_bits, float sa, float sw, float alpha) {
  if constexpr (FMT == kINT8) {
    return (__int2float_rn(static_cast<int>(acc_bits)) * sa) * sw;
  } else if constexpr (FMT == kFP8) {
    return (__uint_as_float(acc_bits) * sa) * sw;
  } else if constexpr (FMT == kNVF4) {
    return __uint_as_float(acc_bits) * alpha;
  } else {
    return __uint_as_float(acc_bits);   // Block_FP8: already promoted
  }
}

template <int FMT>
__device__ __forceinline__ uint32_t add_acc(uint32_t a, uint32_t b) {
  if constexpr (FMT == kINT8) return (uint32_t)((int)a + (int)b);
  else return __float_as_uint(__uint_as_float(a) + __uint_as_float(b));
}

// NVFP4 tensor-scale product; a grouped launch takes expert e's weight
// tensor scale g_w[e] (every expert quantised as its own tensor).
template <int FMT>
__device__ __forceinline__ float alpha_of(const GemmParams& prm, int expert = 0) {
  if constexpr (FMT == kNVF4) return __ldg(prm.g_a) * __ldg(prm.g_w + expert);
  else return 1.f;
}

// Final epilogue of tile element (r, c) = output (m, n).  FP8 / INT8 take
// their per-row scales from the staged copies: row_s[r] is the scale of P row
// r and col_s[c] that of Q row c.
template <int FMT, bool SWAP>
__device__ __forceinline__ void emit(const GemmParams& prm, int r, int c, int m, int n,
                                     uint32_t acc_bits, float alpha, const float* row_s,
                                     const float* col_s) {
  if (prm.out_kind == 1) {
    reinterpret_cast<uint32_t*>(prm.Y)[(size_t)m * prm.ldy + n] = acc_bits;
    return;
  }
  float sa = 1.f, sw = 1.f;
  if constexpr (FMT == kFP8 || FMT == kINT8) {
    sa = SWAP ? col_s[c] : row_s[r];
    sw = SWAP ? row_s[r] : col_s[c];
  }
  reinterpret_cast<__nv_bfloat16*>(prm.Y)[(size_t)m * prm.ldy + n] =
      __float2bfloat16_rn(finish_value<FMT>(acc_bits, sa, sw, alpha));
}

// Scales of the eight consecutive output channels n0 .. n0+7 of tile element
// (r, c) (FP8_Dynamic, W8A8_INT8): the token's scale sa and the channels'
// scales sw[0..7], read from the staged copies as two 16-byte vectors when
// the channel index is a multiple of 8 (it always is in the vector paths).
template <bool SWAP>
__device__ __forceinline__ void scales8(const float* row_s, const float* col_s, int r, int c, float& sa,
                                        float (&sw)[8]) {
  sa = SWAP ? col_s[c] : row_s[r];
  const int ch = SWAP ? r : c;
  const float* s = SWAP ? row_s + r : col_s + c;
  if ((ch & 7) == 0) {
    const float4 a = reinterpret_cast<const float4*>(s)[0];
    const float4 b = reinterpret_cast<const float4*>(s)[1];
    sw[0] = a.x; sw[1] = a.y; sw[2] = a.z; sw[3] = a.w;
    sw[4] = b.x; sw[5] = b.y; sw[6] = b.z; sw[7] = b.w;
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) sw[j] = s[j];
  }
}

// Grouped launches: the token tile of a CTA.  blockIdx.y enumerates the
// token tiles of all experts in expert order (ceil(tokens_e / BN) per expert).
// Lane l owns experts [8 l, 8 l + 8): it sums their tile counts, one warp
// scan turns the sums into each lane's first tile, the lane whose range holds
// blockIdx.y walks its eight experts to the one it falls in.  Offsets come
// from the preceding kernel (routing) and are clamped to [0, M], so a
// malformed routing never leads to an access outside A or y.  Writes {expert
// (-1: no tile), first token, tokens, scale row} to map; the scale row is the
// tile's first token in the NVFP4 per-expert padded scale layout (every
// expert's scale rows start on a 128-row atom boundary: expert e's first
// row is 128 x the sum of ceil(tokens / 128) over the experts before it).
// With SF, a tile whose scale rows would pass the layout's end (only a
// malformed, decreasing routing claims that many atoms) gets no tile.
template <int BN, bool SF>
__device__ __forceinline__ void grouped_tile(const GemmParams& prm, int lane, int* map) {
  constexpr unsigned kFull = 0xffffffffu;
  constexpr int kPer = kMaxExperts / 32;
  const int E = prm.experts;
  const int y = blockIdx.y;
  const int e0 = lane * kPer;
  int ov[kPer + 1];                            // offsets[e0 .. e0 + kPer], past E: offsets[E]
#pragma unroll
  for (int j = 0; j <= kPer; ++j)
    ov[j] = min(max(__ldcg(prm.expert_offsets + min(e0 + j, E)), 0), prm.M);
  int sum = 0;
#pragma unroll
  for (int j = 0; j < kPer; ++j) sum += (max(ov[j + 1] - ov[j], 0) + BN - 1) / BN;
  int incl = sum;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int t = __shfl_up_sync(kFull, incl, d);
    if (lane >= d) incl += t;
  }
  const int excl = incl - sum;
  // 128-row scale atoms of this lane's experts, and the atoms before them
  int asum = 0;
#pragma unroll
  for (int j = 0; j < kPer; ++j) asum += (max(ov[j + 1] - ov[j], 0) + 127) / 128;
  int aincl = asum;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int t = __shfl_up_sync(kFull, aincl, d);
    if (lane >= d) aincl += t;
  }
  const unsigned hit = __ballot_sync(kFull, y >= excl && y < incl);
  if (hit == 0u) {
    if (lane == 0) map[0] = -1;
    return;
  }
  if (lane == __ffs(hit) - 1) {
    int base = excl;
    int abase = aincl - asum;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int cnt = max(ov[j + 1] - ov[j], 0);
      const int t = (cnt + BN - 1) / BN;
      if (y < base + t) {
        const int tile = y - base;
        map[0] = e0 + j;
        map[1] = ov[j] + tile * BN;
        map[2] = min(BN, cnt - tile * BN);
        map[3] = abase * 128 + tile * BN;
        if constexpr (SF) {
          const int a = min(E, prm.M);
          if (map[3] + map[2] > ((prm.M - a) / 128 + a) * 128) map[0] = -1;
        }
        break;
      }
      base += t;
      abase += (cnt + 127) / 128;
    }
  }
}

template <int FMT, bool SWAP, int BN, bool FUSED, bool GROUPED>
__global__ void __launch_bounds__(Cfg<FMT, BN>::kThreads, Cfg<FMT, BN>::kMinBlocks)
    qgemm_kernel(const __grid_constant__ CUtensorMap tmap_p,
                 const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_y,
                 const GemmParams prm) {
  using C = Cfg<FMT, BN>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // Fused activation quantisation is its own instantiation, so the TMA-fed
  // kernel carries none of its code.
  constexpr bool kFusable = FUSED && SWAP && FMT != kNVF4;
  constexpr bool fused = kFusable;
  constexpr bool kDualAble = dual_issue_able<FMT, SWAP, BN, FUSED, GROUPED>();
  constexpr int kTmemAlloc = tmem_cols<FMT, SWAP, BN, FUSED, GROUPED>();
  constexpr bool a_threads = fused;                    // Q tiles written by the epilogue warps
  const SmemLayout L =
      smem_layout<FMT, SWAP, BN>(prm.stages, prm.nkt_max, prm.recv_cols, a_threads ? prm.nkt_max : 0);
  const int S = prm.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;
  uint64_t* tfull = acc_full + 1;
  uint64_t* tempty = tfull + 4;
  uint64_t* recv_full = tempty + 4;
  uint64_t* amax_full = recv_full + 1;
  uint64_t* act_ready = amax_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc);
  volatile int* flag_last = reinterpret_cast<volatile int*>(smem + L.misc + 4);
  volatile int* flag_abort = reinterpret_cast<volatile int*>(smem + L.misc + 8);
  volatile int* flag_epi = reinterpret_cast<volatile int*>(smem + L.misc + 12);
  float* row_s = reinterpret_cast<float*>(smem + L.epis);
  float* col_s = row_s + 128;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int p0 = blockIdx.x * 128;
  int q0 = blockIdx.y * BN;
  // tokens of this CTA are [q0, Mlim); weight rows start at wrow (grouped:
  // the expert's first row)
  int Mlim = prm.M;
  int wrow = 0;
  int sf_row_q = q0;                           // NVFP4: scale row of the first Q row of the tile
  int expert = 0;
  if constexpr (GROUPED) {
    // which expert and tokens this CTA serves depends on the routing of the
    // preceding kernel: resolved before any set-up, and a CTA without work
    // leaves at once (all CTAs of a split-K cluster share the tile)
    __shared__ int gmap[4];
    griddep_wait();
    if (warp == 0) grouped_tile<BN, FMT == kNVF4>(prm, lane, gmap);
    __syncthreads();
    if (gmap[0] < 0 || gmap[2] <= 0) return;
    q0 = gmap[1];
    Mlim = gmap[1] + gmap[2];
    wrow = gmap[0] * prm.N;
    sf_row_q = gmap[3];
    expert = gmap[0];
  }
  const int kz = blockIdx.z;
  // split_k is a power of two: slice z is K tiles [z kt / split_k, (z + 1) kt / split_k)
  const int sk_log2 = __ffs(prm.split_k) - 1;
  const int kt_begin = (int)(((long long)kz * prm.kt_total) >> sk_log2);
  const int kt_end = (int)(((long long)(kz + 1) * prm.kt_total) >> sk_log2);
  const int nkt = kt_end - kt_begin;
  if (threadIdx.x == 0) trace_at(prm, kTrEntry);
  const bool cluster_red = prm.split_k > 1 && prm.reduce_mode == kReduceCluster;
  bool epi_phase1 = false;                                 // epilogue warps waited cluster phase 1
  const int rows_per = 128 / prm.split_k;                  // cluster mode: rows owned per CTA
  // two MMA issuers: the ring holds every K tile of the slice (no refills)
  const bool dual = kDualAble && prm.stages >= nkt && nkt >= 2;
  const uint32_t slot_bytes = 4u * (uint32_t)(rows_per * prm.recv_cols);

  if (threadIdx.x == 0) {
    prefetch_tmap(&tmap_p);
    prefetch_tmap(&tmap_q);
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(acc_full, dual ? 2 : 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], C::kEpiWarps);
    }
    // push mode: one arrival (the receiver's expected byte count); the
    // senders' asynchronous stores complete the bytes
    mbar_init(recv_full, 1);
    // fused per-token amax exchange: one arrival (the receiver's expected
    // byte count); the peers' asynchronous stores complete the bytes
    mbar_init(amax_full, 1);
    // thread-written activation slice: one arrival per epilogue thread
    mbar_init(act_ready, C::kEpiThreads);
    *flag_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemAlloc);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  if (threadIdx.x == 0) trace_at(prm, kTrReady);
  // Cluster phase 1 (arrive now, wait before the first remote access): the
  // barriers of every CTA in the cluster are initialised.
  if (cluster_red) cluster_arrive();
  // Let the next kernel of the stream start its prologue; it waits on our
  // completion before touching what we write.
  if (threadIdx.x == 0) griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && nkt > 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_a = policy_evict_last();
      const CUtensorMap* map_w = SWAP ? &tmap_p : &tmap_q;
      const CUtensorMap* map_a = SWAP ? &tmap_q : &tmap_p;
      const uint32_t off_w = SWAP ? L.p : L.q;
      const uint32_t off_a = SWAP ? L.q : L.p;
      const uint32_t bytes_w = SWAP ? kPTileBytes : C::kQTileBytes;
      const uint32_t bytes_a = SWAP ? C::kQTileBytes : kPTileBytes;
      const int row_w = SWAP ? wrow + p0 : q0;
      const int row_a = SWAP ? q0 : p0;
      // NVFP4 scale atoms: P rows [p0, p0+128) are one 128-row block; Q has
      // one or two blocks (the second only if it holds any row).
      const int sfq_atoms = (C::kSfQAtoms == 2 && q0 + 128 < (GROUPED ? Mlim : prm.rows_q)) ? 2 : 1;
      const uint32_t stage_tx = a_threads ? bytes_w
                                      : kPTileBytes + C::kQTileBytes +
                                            (C::kNvf4 ? (uint32_t)(4 * kSfAtomBytes * (1 + sfq_atoms)) : 0u);
      auto load_w = [&](int i, int st) {
        const int kt = kt_begin + i;
        tma_load_2d(smem + off_w + st * bytes_w, map_w, &full[st], kt * kKTileBytes, row_w, pol_w);
        if constexpr (C::kNvf4) {
          const uint8_t* sfw = SWAP ? prm.sf_p : prm.sf_q;
          const int rb = row_w / 128;
          if (SWAP) {
            bulk_load(smem + L.sfp + st * C::kSfPBytes,
                      sfw + ((size_t)rb * prm.sf_atoms_per_rb + kt * 4) * kSfAtomBytes,
                      4 * kSfAtomBytes, &full[st]);
          } else {
            for (int a = 0; a < sfq_atoms; ++a)
              bulk_load(smem + L.sfq + st * C::kSfQBytes + a * 4 * kSfAtomBytes,
                        sfw + ((size_t)(rb + a) * prm.sf_atoms_per_rb + kt * 4) * kSfAtomBytes,
                        4 * kSfAtomBytes, &full[st]);
          }
        }
      };
      auto load_a = [&](int i, int st) {
        const int kt = kt_begin + i;
        tma_load_2d(smem + off_a + st * bytes_a, map_a, &full[st], kt * kKTileBytes, row_a, pol_a);
        if constexpr (C::kNvf4) {
          const uint8_t* sfa = SWAP ? prm.sf_q : prm.sf_p;
          const int rb = (SWAP ? sf_row_q : row_a) / 128;
          if (SWAP) {
            for (int a = 0; a < sfq_atoms; ++a)
              bulk_load(smem + L.sfq + st * C::kSfQBytes + a * 4 * kSfAtomBytes,
                        sfa + ((size_t)(rb + a) * prm.sf_atoms_per_rb + kt * 4) * kSfAtomBytes,
                        4 * kSfAtomBytes, &full[st]);
          } else {
            bulk_load(smem + L.sfp + st * C::kSfPBytes,
                      sfa + ((size_t)rb * prm.sf_atoms_per_rb + kt * 4) * kSfAtomBytes,
                      4 * kSfAtomBytes, &full[st]);
          }
        }
      };
      const int pre = nkt < S ? nkt : S;
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(&full[i], stage_tx);
        load_w(i, i);
        if (i == 0) trace_at(prm, kTrFirstLoad);
      }
      if constexpr (SWAP && !GROUPED) {
        if (prm.l2_ahead > 0) {
          // the weight slice of the CTA l2_ahead places later in launch
          // order: clusters launch whole (cluster index x + y * gx, the
          // split slices z inside), plain grids in x, y, z order
          const int gx = gridDim.x, gy = gridDim.y, gz = gridDim.z;
          int tx = -1, tz = 0;
          if (cluster_red) {
            const int tc = blockIdx.x + gx * blockIdx.y + prm.l2_ahead;
            if (tc < gx * gy) { tx = tc % gx; tz = kz; }
          } else {
            // the launch keeps l2_ahead at 0 unless gx * gy * gz fits 31 bits
            const unsigned t = blockIdx.x + (unsigned)gx * (blockIdx.y + (unsigned)gy * kz) + (unsigned)prm.l2_ahead;
            if (t < (unsigned)(gx * gy * gz)) { tx = (int)(t % (unsigned)gx); tz = (int)(t / (unsigned)(gx * gy)); }
          }
          if (tx >= 0) {
            const int t_begin = (int)(((long long)tz * prm.kt_total) >> sk_log2);
            const int t_end = (int)(((long long)(tz + 1) * prm.kt_total) >> sk_log2);
            for (int kt = t_begin; kt < t_end; ++kt) {
              tma_prefetch_l2_2d(map_w, kt * kKTileBytes, tx * 128);
              if constexpr (C::kNvf4)
                bulk_prefetch_l2(prm.sf_p + ((size_t)tx * prm.sf_atoms_per_rb + kt * 4) * kSfAtomBytes,
                                 4 * kSfAtomBytes);
            }
          }
        }
      }
      if (!a_threads) {                        // activations come from the preceding kernel
        griddep_wait();
        trace_at(prm, kTrDepWait);
        for (int i = 0; i < pre; ++i) load_a(i, i);
      }
      bool ok = true;
      int issued = pre;
      int st = 0;                              // stage of K tile i; its previous use's phase
      uint32_t ph = 0;
      for (int i = pre; i < nkt; ++i) {
        if (!mbar_wait(&empty[st], ph, prm.err, prm.wait_ns)) { ok = false; break; }
        mbar_arrive_expect_tx(&full[st], stage_tx);
        load_w(i, st);
        if (!a_threads) load_a(i, st);
        issued = i + 1;
        if (++st == S) { st = 0; ph ^= 1u; }
      }
      if constexpr (kDualAble) {
        if (dual) {
          // second MMA issuer: the odd K tiles into the second accumulator
          // (every tile has its own stage, filled once: phase 0)
          const uint64_t dp0 = sdesc_sw128(smem_u32(smem + L.p));
          const uint64_t dq0 = sdesc_sw128(smem_u32(smem + L.q));
          const uint32_t d_t = tmem_base + (uint32_t)BN;
          // fused: the activation tiles are written by the epilogue warps
          bool issued_all = !a_threads || mbar_wait(act_ready, 0, prm.err, prm.wait_ns);
          for (int i = 1; i < nkt && issued_all; i += 2) {
            if (!mbar_wait(&full[i], 0, prm.err, prm.wait_ns)) { issued_all = false; break; }
            tc_fence_after();
            const uint64_t dp = dp0 + (uint64_t)((i * kPTileBytes) >> 4);
            const uint64_t dq = dq0 + (uint64_t)((i * C::kQTileBytes) >> 4);   // stage i, or act tile i
#pragma unroll
            for (int s = 0; s < 4; ++s) {
              const uint32_t accum = (i > 1 || s > 0);
              if constexpr (FMT == kINT8) mma_i8(d_t, dp + (uint64_t)(2 * s), dq + (uint64_t)(2 * s), C::kIdesc, accum);
              else mma_f8f6f4(d_t, dp + (uint64_t)(2 * s), dq + (uint64_t)(2 * s), C::kIdesc, accum);
            }
          }
          if (!issued_all) *flag_abort = 1;
          mma_commit(acc_full);
        }
      }
      if (!ok) {
        *flag_abort = 1;
        // Drain: wait (bounded) until every issued copy has landed.
        for (int i = (issued > S ? issued - S : 0); i < issued; ++i)
          mbar_wait(&full[i % S], (i / S) & 1, prm.err, prm.wait_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0 && nkt > 0) {
      // One k tile costs this thread a barrier test, four MMA issues and a
      // commit; everything else is kept out of the loop.  Descriptors are
      // built once for stage 0 / K step 0: a stage or K step adds its byte
      // offset / 16 to the start-address field (bits 0-13, which shared
      // addresses below 256 KB never carry out of).
      const uint64_t dp0 = sdesc_sw128(smem_u32(smem + L.p));
      const uint64_t dq0 = sdesc_sw128(smem_u32(smem + L.q));
      const uint64_t dsfp0 = sdesc_plain_32x16(smem_u32(smem + L.sfp));
      const uint64_t dsfq0 = sdesc_plain_32x16(smem_u32(smem + L.sfq));
      const uint32_t sfa_t = tmem_base + C::kSfaCol;
      const uint32_t sfb_t = tmem_base + C::kSfbCol;
      // word offset of this CTA's first Q row inside its 128-row SF atom
      const uint32_t sfb_word = (uint32_t)((sf_row_q % 128) / 32);
      int st = 0;                              // stage of K tile i, and its full-barrier phase
      uint32_t ph = 0;
      int gb = 0, gr = 0;                      // Block_FP8: group buffer of K tile i, and its round
      bool abort = false;
      const int istep = dual ? 2 : 1;          // two issuers: this thread takes the even K tiles
      for (int i = 0; i < nkt; i += istep) {
        if (dual) st = i;                      // one stage per K tile, phase 0
        if (!mbar_wait(&full[st], ph, prm.err, prm.wait_ns)) { abort = true; break; }
        if (i == 0) {
          if (a_threads && !mbar_wait(act_ready, 0, prm.err, prm.wait_ns)) { abort = true; break; }
          trace_at(prm, kTrFirstFull);
        }
        if (i == nkt - 1) trace_at(prm, kTrLastFull);
        uint32_t d_t = tmem_base;
        if constexpr (C::kBlock) {
          if (gr > 0 && !mbar_wait(&tempty[gb], (uint32_t)(gr - 1) & 1u, prm.err, prm.wait_ns)) { abort = true; break; }
          d_t = tmem_base + (uint32_t)(gb * BN);
        }
        tc_fence_after();
        const uint64_t dp = dp0 + (uint64_t)((st * kPTileBytes) >> 4);
        const uint64_t dq = dq0 + (uint64_t)(((a_threads ? i : st) * C::kQTileBytes) >> 4);
        if constexpr (C::kNvf4) {
          const uint64_t sfp = dsfp0 + (uint64_t)((st * C::kSfPBytes) >> 4);
          const uint64_t sfq = dsfq0 + (uint64_t)((st * C::kSfQBytes) >> 4);
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            tmem_cp_32x128b_x4(sfa_t + 4 * s, sfp + (uint64_t)((s * kSfAtomBytes) >> 4));
#pragma unroll
            for (int a = 0; a < C::kSfQAtoms; ++a)
              tmem_cp_32x128b_x4(sfb_t + 4 * C::kSfQAtoms * s + 4 * a,
                                 sfq + (uint64_t)((a * 4 * kSfAtomBytes + s * kSfAtomBytes) >> 4));
          }
        }
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint64_t da = dp + (uint64_t)(2 * s);   // 32 bytes further along K
          const uint64_t db = dq + (uint64_t)(2 * s);
          const uint32_t accum = C::kBlock ? (s > 0) : (i > 0 || s > 0);
          if constexpr (C::kNvf4)
            mma_nvf4(d_t, da, db, C::kIdesc, sfa_t + 4 * s,
                     sfb_t + 4 * C::kSfQAtoms * s + sfb_word, accum);
          else if constexpr (FMT == kINT8)
            mma_i8(d_t, da, db, C::kIdesc, accum);
          else
            mma_f8f6f4(d_t, da, db, C::kIdesc, accum);
        }
        mma_commit(&empty[st]);
        if constexpr (C::kBlock) {
          mma_commit(&tfull[gb]);
          if (++gb == C::kNAcc) { gb = 0; ++gr; }
        }
        if (++st == S) { st = 0; ph ^= 1u; }
      }
      if (abort) *flag_abort = 1;
      if constexpr (!C::kBlock) mma_commit(acc_full);
      trace_at(prm, kTrLastMma);
    }
  } else {
    // --------------------------------------------------------------- epilogue
    constexpr int ET = C::kEpiThreads;
    constexpr int NC = C::kCols;
    constexpr int CW = NC >= 32 ? 32 : NC;     // accumulator columns per TMEM load
    const int quarter = warp & 3;              // TMEM lanes this warp may access
    const int row = quarter * 32 + lane;       // row of P in the tile
    const int etid = threadIdx.x - 64;         // 0..ET-1
    const int cbeg = ((warp - 2) / 4) * NC;    // this thread's columns [cbeg, cbeg + NC)
    const uint32_t lane_addr = tmem_base + ((uint32_t)(quarter * 32) << 16);

    // ---- fused activation slice (Swap-AB): the bf16 activations of tokens
    // [q0, q0 + Mt) x K tiles [kt_begin, kt_begin + nkt), quantised into the
    // dedicated Q region, K tile j at L.q + j * BN * 128, every byte where a TMA copy
    // with the 128-byte swizzle would have put it (16-byte chunk index XOR
    // row % 8).  The loads of a batch are all in flight together (L2 only:
    // the preceding kernel wrote them); each epilogue thread then arrives
    // once on act_ready, after a proxy fence that makes its writes visible
    // to the tensor core.
    const int Mt = min(BN, prm.M - q0);                      // real tokens of this tile
    uint8_t* const qtiles = smem + L.q;
    uint32_t* const amax_u = reinterpret_cast<uint32_t*>(smem + L.fuse);   // [BN]
    float* const exch = reinterpret_cast<float*>(smem + L.fuse) + BN;      // [split][BN]
    float* const sa_blk = reinterpret_cast<float*>(smem + L.scales);       // Block_FP8 act scales
    const uint4 zero4 = make_uint4(0u, 0u, 0u, 0u);
    // fused units: 8 elements = 16 bytes of bf16 -> 8 code bytes; unit u is
    // K tile u / (Mt*16), token row (u % (Mt*16)) / 16, elements 8*(u % 16)..
    const int UT = Mt * 16;
    auto unit_load = [&](int u) -> uint4 {
      const int j = u / UT, rem = u - j * UT;
      const int k = (kt_begin + j) * kKTileBytes + (rem & 15) * 8;
      if (k >= prm.K) return zero4;
      return __ldcg(reinterpret_cast<const uint4*>(prm.act + (size_t)(q0 + (rem >> 4)) * prm.lda + k));
    };
    auto unit_store = [&](int u, uint2 codes) {
      const int j = u / UT, rem = u - j * UT;
      const int r = rem >> 4, c8 = rem & 15;
      const uint32_t off = (uint32_t)(j * C::kQTileBytes + r * kKTileBytes) +
                           ((uint32_t)(((c8 >> 1) ^ (r & 7)) << 4) | (uint32_t)((c8 & 1) << 3));
      *reinterpret_cast<uint2*>(qtiles + off) = codes;
    };
    auto publish_act = [&]() {
      fence_proxy_async_smem();
      mbar_arrive(act_ready);
      if (etid == 0) trace_at(prm, kTrActReady);
    };
    if constexpr (kFusable) {
      if (a_threads) {
        // independent of the preceding kernel: the padding token rows of
        // every K tile are zero, the amax slots start at zero
        const int pad = BN - Mt;
        for (int idx = etid; idx < nkt * pad * 8; idx += ET) {
          const int j = idx / (pad * 8), rem = idx % (pad * 8);
          *reinterpret_cast<uint4*>(qtiles + j * C::kQTileBytes + (Mt + rem / 8) * kKTileBytes +
                                    (rem % 8) * 16) = zero4;
        }
        if (fused && etid < BN) amax_u[etid] = 0u;
        if (fused) named_bar_sync(1, ET);
      }
    }
    // FP8 / INT8 Swap-AB: the weight (row) scales do not depend on the
    // preceding kernel, so they are staged while it still runs
    if constexpr (C::kRowColScales && SWAP)
      for (int r = etid; r < 128; r += ET)
        row_s[r] = (p0 + r < prm.rows_p) ? __ldg(prm.scale_w + wrow + p0 + r) : 0.f;
    griddep_wait();                            // scales/partials/activations of earlier kernels
    // push-mode cluster split-K: wait for cluster phase 1 (every receiver's
    // barriers initialised) now, while the MMAs run, not after the accumulator
    if constexpr (C::kPush && !kFusable) {
      if (cluster_red) {
        cluster_wait();
        epi_phase1 = true;
      }
    }
    if (a_threads && etid == 0) trace_at(prm, kTrDepWait);
    bool fz_ok = true;
    // FP8 / INT8: the remaining per-row scales of this tile (activation
    // scales come from the preceding kernel unless the kernel quantises)
    if constexpr (C::kRowColScales) {
      if constexpr (!SWAP)
        for (int r = etid; r < 128; r += ET) row_s[r] = (p0 + r < prm.rows_p) ? __ldg(prm.scale_a + p0 + r) : 0.f;
      const float* sq = SWAP ? prm.scale_a : prm.scale_w;
      if (!fused)
        for (int c = etid; c < BN; c += ET) col_s[c] = (q0 + c < prm.rows_q) ? __ldg(sq + q0 + c) : 0.f;
    }
    if constexpr (kFusable && C::kRowColScales) {
      if (fused) {
        // ---- per-token FP8 / INT8.  Pass 1: amax of every token row over
        // this slice (the first kCache units of a thread stay in registers).
        constexpr bool kI8 = FMT == kINT8;
        constexpr int kCache = 8;
        const int U = nkt * UT;
        uint4 cache[kCache];
#pragma unroll
        for (int b = 0; b < kCache; ++b) {
          const int u = b * ET + etid;
          cache[b] = u < U ? unit_load(u) : zero4;
        }
#pragma unroll
        for (int b = 0; b < kCache; ++b) {
          const int u = b * ET + etid;
          if (u < U) {
            float x[8];
            unpack8(cache[b], x);
            atomicMax(&amax_u[(u % UT) >> 4], __float_as_uint(absmax8(x)));
          }
        }
        for (int u0 = kCache * ET; u0 < U; u0 += 4 * ET) {     // beyond the cache: 4 loads in flight
          uint4 v[4];
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const int u = u0 + b * ET + etid;
            v[b] = u < U ? unit_load(u) : zero4;
          }
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const int u = u0 + b * ET + etid;
            if (u < U) {
              float x[8];
              unpack8(v[b], x);
              atomicMax(&amax_u[(u % UT) >> 4], __float_as_uint(absmax8(x)));
            }
          }
        }
        named_bar_sync(1, ET);
        if (etid == 0) trace_at(prm, kTrActLoaded);
        // the row amax spans the whole K: the split-K CTAs of the cluster
        // swap their partial maxima (thread etid serves peer etid % split)
        if (cluster_red) {
          const int Sk = prm.split_k;
          // every CTA of the cluster sends this one its Mt maxima
          if (etid == 0) mbar_arrive_expect_tx(amax_full, (uint32_t)(Sk * Mt * 4));
          cluster_wait();                      // phase 1: every peer is initialised
          epi_phase1 = true;
          const uint32_t z = (uint32_t)(etid % Sk);
          const uint32_t dst = mapa_shared(smem_u32(exch + kz * BN), z);
          const uint32_t zbar = mapa_shared(smem_u32(amax_full), z);
          for (int r = etid / Sk; r < Mt; r += ET / Sk) st_async_b32(dst + 4u * (uint32_t)r, amax_u[r], zbar);
          fz_ok = mbar_wait_cluster(amax_full, 0, prm.err, prm.wait_ns);
        }
        if (etid == 0) trace_at(prm, kTrActAmax);
        if (etid < BN) {
          float am = 0.f;
          if (etid < Mt) {
            if (cluster_red) {
              for (int zz = 0; zz < prm.split_k; ++zz) am = fmaxf(am, exch[zz * BN + etid]);
            } else {
              am = __uint_as_float(amax_u[etid]);
            }
          }
          const float sc = scale_of_amax<kI8>(am);
          col_s[etid] = etid < Mt ? sc : 0.f;
          if (etid < Mt && prm.act_scale_out != nullptr && blockIdx.x == 0 && kz == 0)
            prm.act_scale_out[q0 + etid] = sc;
        }
        named_bar_sync(1, ET);
        // pass 2: the codes of every unit
#pragma unroll
        for (int b = 0; b < kCache; ++b) {
          const int u = b * ET + etid;
          if (u < U) {
            float x[8];
            unpack8(cache[b], x);
            const float sc = col_s[(u % UT) >> 4];
            unit_store(u, quant8<kI8>(x, sc));
          }
        }
        for (int u0 = kCache * ET; u0 < U; u0 += 4 * ET) {
          uint4 v[4];
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const int u = u0 + b * ET + etid;
            v[b] = u < U ? unit_load(u) : zero4;
          }
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const int u = u0 + b * ET + etid;
            if (u < U) {
              float x[8];
              unpack8(v[b], x);
              unit_store(u, quant8<kI8>(x, col_s[(u % UT) >> 4]));
            }
          }
        }
        publish_act();
      }
    }
    if constexpr (kFusable && C::kBlock) {
      if (fused) {
        // ---- Block_FP8: 1x128 groups are local to a K tile; a group is 16
        // consecutive units on 16 consecutive lanes (ET and UT are multiples
        // of 16), its amax a max over shuffles.  Rounds are uniform over the
        // epilogue threads, four units of loads in flight per thread.
        const int U = nkt * UT;
        const int rounds = (U + ET - 1) / ET;
        for (int b0 = 0; b0 < rounds; b0 += 4) {
          uint4 v[4];
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const int u = (b0 + b) * ET + etid;
            v[b] = (b0 + b < rounds && u < U) ? unit_load(u) : zero4;
          }
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            if (b0 + b < rounds) {
              const int u = (b0 + b) * ET + etid;
              float x[8];
              unpack8(v[b], x);
              float a = absmax8(x);
#pragma unroll
              for (int o = 8; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
              const float sc = scale_of_amax<false>(a);
              if (u < U) {
                unit_store(u, quant8<false>(x, sc));
                const int j = u / UT, rem = u - j * UT;
                if ((rem & 15) == 0) {
                  sa_blk[(rem >> 4) * nkt + j] = sc;
                  if (prm.act_scale_out != nullptr && blockIdx.x == 0)
                    prm.act_scale_out[(size_t)(q0 + (rem >> 4)) * prm.groups + kt_begin + j] = sc;
                }
              }
            }
          }
        }
        publish_act();
      }
    }
    bool ok = true;                            // warp-uniform
    // Block_FP8 promoted accumulator, as packed fp32 pairs: the promotion is
    // one fma.rn.f32x2 per two elements (two independent round-to-nearest
    // FMAs, the same bits as fmaf), halving the FMA issue slots it takes
    uint64_t acc2[NC / 2];
    if constexpr (C::kBlock) {
      float* sa_s = reinterpret_cast<float*>(smem + L.scales);          // act scales
      constexpr int act_rows = block_act_rows<SWAP, BN>();
      float* sw_s = sa_s + act_rows * prm.nkt_max;                      // weight scales
      const int G = prm.groups;
      const int g0 = kt_begin;
      // Stage this CTA's scales: activations per (row, group), weights per
      // (128-row block, group).
      const int act_base = SWAP ? q0 : p0;
      if (!fused) {
        for (int idx = etid; idx < act_rows * nkt; idx += ET) {
          const int r = idx / nkt, gl = idx % nkt;
          const int m = act_base + r;
          sa_s[idx] = (m < prm.M) ? __ldg(prm.scale_a + (size_t)m * G + g0 + gl) : 0.f;
        }
      } else {
        // fused: rows of real tokens were written above; padding tokens
        // scale to zero
        for (int idx = Mt * nkt + etid; idx < act_rows * nkt; idx += ET) sa_s[idx] = 0.f;
      }
      constexpr int WB = block_weight_blocks<SWAP, BN>();              // weight blocks per tile
      const int wrow0 = (SWAP ? p0 : q0) / 128;                        // block within the weight
      const int nblk = (prm.N + 127) / 128;
      for (int idx = etid; idx < WB * nkt; idx += ET) {
        const int gl = idx / WB, jb = idx % WB;
        const int b = wrow0 + jb;
        sw_s[idx] = (b < nblk) ? __ldg(prm.scale_w + (size_t)(wrow / 128 + b) * G + g0 + gl) : 0.f;
      }
      named_bar_sync(1, ET);
#pragma unroll
      for (int c = 0; c < NC / 2; ++c) acc2[c] = 0ull;
      ok = __all_sync(0xffffffffu, fz_ok);
      for (int i = 0; i < nkt && ok; ++i) {
        const int b = i % C::kNAcc;
        ok = __all_sync(0xffffffffu, mbar_wait(&tfull[b], (i / C::kNAcc) & 1, prm.err, prm.wait_ns));
        if (!ok) break;
        tc_fence_after();
        // acc += p_g * (s_a * s_w): one FMA per element
        float f_row = 0.f;
        if (!SWAP) f_row = sa_s[row * nkt + i];
        // columns per TMEM round trip: 64 (two loads, one wait) while the
        // accumulator is small, 32 when it already holds 128 registers
        // (16 columns when 16 warps share the register file)
        constexpr int PB = C::kEpiWarps >= 16 ? 16 : NC >= 128 ? 32 : 64;
        constexpr int NCH = (NC + PB - 1) / PB;
        auto ld_chunk = [&](int c0, uint32_t (&v)[PB]) {
          if constexpr (NC % 32 == 0 && PB >= 32) {
            tmem_ld32(lane_addr + b * BN + cbeg + c0, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
            if constexpr (PB == 64)
              if (c0 + 32 < NC)
                tmem_ld32(lane_addr + b * BN + cbeg + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
          } else {                             // 16-column tiles: stay inside the buffer
            tmem_ld16(lane_addr + b * BN + cbeg + c0, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
          }
        };
        auto fma_chunk = [&](int c0, const uint32_t (&v)[PB]) {
          if (SWAP) {
            const float sw = sw_s[i];
#pragma unroll
            for (int j = 0; j < PB && c0 + j < NC; j += 2)
              ffma2(acc2[(c0 + j) / 2], v[j], v[j + 1],
                    pack_f32x2(sa_s[(cbeg + c0 + j) * nkt + i] * sw, sa_s[(cbeg + c0 + j + 1) * nkt + i] * sw));
          } else {
            // one weight block per chunk (chunks start on multiples of PB
            // and never cross a 128-column block): one scale for all of it
            const float f = f_row * sw_s[i * WB + (WB == 2 ? (cbeg + c0) / 128 : 0)];
            const uint64_t f2 = pack_f32x2(f, f);
#pragma unroll
            for (int j = 0; j < PB && c0 + j < NC; j += 2) ffma2(acc2[(c0 + j) / 2], v[j], v[j + 1], f2);
          }
        };
        if constexpr (NCH >= 2 && PB <= 16) {
          // narrow chunks (16 warps share the register file): the next
          // chunk's TMEM load is in flight while this chunk's FMAs run
          uint32_t va[PB], vb[PB];
          ld_chunk(0, va);
          tmem_ld_wait();
#pragma unroll
          for (int ch = 0; ch < NCH; ch += 2) {
            if (ch + 1 < NCH) ld_chunk((ch + 1) * PB, vb);
            fma_chunk(ch * PB, va);
            if (ch + 1 < NCH) {
              tmem_ld_wait();
              if (ch + 2 < NCH) ld_chunk((ch + 2) * PB, va);
              fma_chunk((ch + 1) * PB, vb);
              if (ch + 2 < NCH) tmem_ld_wait();
            }
          }
        } else {
#pragma unroll
          for (int c0 = 0; c0 < NC; c0 += PB) {
            uint32_t v[PB];
            ld_chunk(c0, v);
            tmem_ld_wait();
            fma_chunk(c0, v);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[b]);
      }
    } else {
      ok = __all_sync(0xffffffffu, fz_ok && mbar_wait(acc_full, 0, prm.err, prm.wait_ns));
      tc_fence_after();
    }
    if (etid == 0) {
      *flag_epi = 0;
      trace_at(prm, kTrAccReady);
    }
    named_bar_sync(1, ET);                     // also publishes the staged scales
    if (!ok) *flag_epi = 1;
    named_bar_sync(1, ET);
    const bool epi_ok = (*flag_epi == 0);      // uniform over the epilogue threads

    const bool split = prm.split_k > 1;
    const int prow = p0 + row;                 // global row of P
    const bool prow_ok = prow < prm.rows_p;
    const size_t MN = (size_t)prm.M * prm.N;
    uint32_t* part = reinterpret_cast<uint32_t*>(prm.partial);
    uint32_t* stage_buf = reinterpret_cast<uint32_t*>(smem + L.p);   // ring, idle now
    const float alpha = alpha_of<FMT>(prm, expert);
    // Accumulator columns [cbeg + c0, cbeg + c0 + CW) of this thread's row.
    auto load_chunk = [&](int c0, uint32_t (&v)[CW]) {
      if constexpr (C::kBlock) {
#pragma unroll
        for (int j = 0; j < CW; j += 2) unpack_u32x2(acc2[(c0 + j) / 2], v[j], v[j + 1]);
      } else if constexpr (CW == 32) {
        tmem_ld32(lane_addr + cbeg + c0, v);
        if constexpr (kDualAble) {
          if (dual) {                          // the second issuer's accumulator
            uint32_t v2[CW];
            tmem_ld32(lane_addr + BN + cbeg + c0, v2);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < CW; ++j) v[j] = add_acc<FMT>(v[j], v2[j]);
          }
        }
        tmem_ld_wait();
      } else {
        tmem_ld16(lane_addr + cbeg + c0, v);
        if constexpr (kDualAble) {
          if (dual) {
            uint32_t v2[CW];
            tmem_ld16(lane_addr + BN + cbeg + c0, v2);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < CW; ++j) v[j] = add_acc<FMT>(v[j], v2[j]);
          }
        }
        tmem_ld_wait();
      }
    };

    // Output tile in the idle ring: raw accumulator bits of tile element
    // (r, c) at otile[tile_index(r, c)], written out by one compact loop that
    // scales, converts and stores 16-byte vectors along the contiguous
    // dimension of y (channels: r under Swap-AB, c otherwise).
    uint32_t* otile = stage_buf;
    // Eight consecutive output channels n0 .. n0+7 of output row m (tile
    // row r / column c): raw accumulators, or scaled, rounded to bf16 and
    // stored as one 16-byte vector where the row pitch allows it.
    auto store8 = [&](int r, int c, int m, int n0, const uint32_t (&acc8)[8]) {
      const bool vec = (prm.ldy % 8) == 0;
      if (prm.out_kind == 1) {
        uint32_t* Yu = reinterpret_cast<uint32_t*>(prm.Y) + (size_t)m * prm.ldy;
        for (int j = 0; j < 8 && n0 + j < prm.N; ++j) Yu[n0 + j] = acc8[j];
        return;
      }
      float y8[8];
      float sa = 1.f, sw[8] = {1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f};
      if constexpr (FMT == kFP8 || FMT == kINT8) scales8<SWAP>(row_s, col_s, r, c, sa, sw);
#pragma unroll
      for (int j = 0; j < 8; ++j) y8[j] = finish_value<FMT>(acc8[j], sa, sw[j], alpha);
      __nv_bfloat16* Yb = reinterpret_cast<__nv_bfloat16*>(prm.Y) + (size_t)m * prm.ldy;
      if (vec && n0 + 8 <= prm.N) {
        uint32_t p[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(y8[2 * h], y8[2 * h + 1]);
          p[h] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        *reinterpret_cast<uint4*>(Yb + n0) = make_uint4(p[0], p[1], p[2], p[3]);
      } else {
        for (int j = 0; j < 8 && n0 + j < prm.N; ++j) Yb[n0 + j] = __float2bfloat16_rn(y8[j]);
      }
    };
    // A thread takes kUB units per round: their shared-memory reads are all
    // issued before the first unit is scaled and stored, so that one warp
    // per TMEM quarter keeps several units in flight.
    auto write_out = [&](int r_begin, int r_count, int c_begin, int c_count) {
      constexpr int kUB = C::kMinBlocks >= 3 ? 2 : 4;
      const int per = SWAP ? r_count / 8 : c_count / 8;          // units per tile column / row
      const int units = SWAP ? c_count * per : r_count * per;
#pragma unroll 1
      for (int u0 = etid; u0 < units; u0 += kUB * ET) {
        uint32_t acc8[kUB][8];
        int rr[kUB], cc[kUB];                  // first of 8 consecutive output channels
#pragma unroll
        for (int k = 0; k < kUB; ++k) {
          const int u = min(u0 + k * ET, units - 1);               // past the end: re-read, never stored
          if (SWAP) { cc[k] = c_begin + u / per; rr[k] = r_begin + (u % per) * 8; }
          else      { rr[k] = r_begin + u / per; cc[k] = c_begin + (u % per) * 8; }
          const uint4* src = reinterpret_cast<const uint4*>(otile + tile_index<SWAP, BN>(rr[k], cc[k]));
          const uint4 w0 = src[0], w1 = src[1];
          acc8[k][0] = w0.x; acc8[k][1] = w0.y; acc8[k][2] = w0.z; acc8[k][3] = w0.w;
          acc8[k][4] = w1.x; acc8[k][5] = w1.y; acc8[k][6] = w1.z; acc8[k][7] = w1.w;
        }
#pragma unroll
        for (int k = 0; k < kUB; ++k) {
          if (u0 + k * ET >= units) break;
          const int m = SWAP ? q0 + cc[k] : p0 + rr[k];
          const int n0 = SWAP ? p0 + rr[k] : q0 + cc[k];
          if (m < Mlim && n0 < prm.N) store8(rr[k], cc[k], m, n0, acc8[k]);
        }
      }
    };

    bool tma_out = false;                      // the tile went out through the y tensor map
    if constexpr (!SWAP && BN >= 64) {
      if (!split && prm.y_tma && epi_ok) {
        // ---- direct, TMA store: each thread scales, rounds and writes its
        // row's channels into 64-channel boxes of 128 rows x 128 bytes (the
        // ring is idle: every MMA has completed); 16-byte chunk k of row r
        // of a box sits at chunk k ^ (r % 8), the TMA 128-byte swizzle, so a
        // quarter warp's eight rows hit eight different bank groups.
        uint8_t* ybuf = smem + L.p;
        float sa = 1.f;
        if constexpr (FMT == kFP8 || FMT == kINT8) sa = row_s[row];
#pragma unroll
        for (int c0 = 0; c0 < NC; c0 += CW) {
          uint32_t v[CW];
          load_chunk(c0, v);
#pragma unroll
          for (int j = 0; j < CW; j += 8) {
            const int col = cbeg + c0 + j;     // a multiple of 8
            float sw[8] = {1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f};
            if constexpr (FMT == kFP8 || FMT == kINT8) {
              const float4 a = reinterpret_cast<const float4*>(col_s + col)[0];
              const float4 b = reinterpret_cast<const float4*>(col_s + col)[1];
              sw[0] = a.x; sw[1] = a.y; sw[2] = a.z; sw[3] = a.w;
              sw[4] = b.x; sw[5] = b.y; sw[6] = b.z; sw[7] = b.w;
            }
            uint32_t pk[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const __nv_bfloat162 b2 =
                  __floats2bfloat162_rn(finish_value<FMT>(v[j + 2 * h], sa, sw[2 * h], alpha),
                                        finish_value<FMT>(v[j + 2 * h + 1], sa, sw[2 * h + 1], alpha));
              pk[h] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            const uint32_t off = (uint32_t)(col >> 6) * 16384u + (uint32_t)row * 128u +
                                 ((uint32_t)(((col & 63) >> 3) ^ (row & 7)) << 4);
            *reinterpret_cast<uint4*>(ybuf + off) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
        fence_proxy_async_smem();
        named_bar_sync(1, ET);
        if (etid == 0) {
#pragma unroll
          for (int b = 0; b < BN / 64; ++b) tma_store_2d(&tmap_y, ybuf + b * 16384, (q0 + b * 64) * 2, p0);
          bulk_commit();
          bulk_wait_all();
        }
        tma_out = true;
      }
    }
    if (tma_out) {
    } else if (!split) {
      // ---- direct: accumulator -> tile -> y
      if constexpr (!C::kBlock && !SWAP && CW == 32 && NC >= 128) {
        // wide rows: the next 32 columns' TMEM load is in flight while this
        // chunk goes to the tile
        if (epi_ok) {
          auto put = [&](int c0, const uint32_t (&v)[32]) {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              *reinterpret_cast<uint4*>(otile + tile_index<SWAP, BN>(row, cbeg + c0 + j)) =
                  make_uint4(v[j], v[j + 1], v[j + 2], v[j + 3]);
          };
          uint32_t va[32], vb[32];
          tmem_ld32(lane_addr + cbeg, va);
          tmem_ld_wait();
#pragma unroll
          for (int c0 = 0; c0 < NC; c0 += 64) {
            tmem_ld32(lane_addr + cbeg + c0 + 32, vb);
            put(c0, va);
            tmem_ld_wait();
            if (c0 + 64 < NC) tmem_ld32(lane_addr + cbeg + c0 + 64, va);
            put(c0 + 32, vb);
            if (c0 + 64 < NC) tmem_ld_wait();
          }
        }
      } else if (epi_ok) {
#pragma unroll
        for (int c0 = 0; c0 < NC; c0 += CW) {
          uint32_t v[CW];
          load_chunk(c0, v);
          if constexpr (SWAP) {
#pragma unroll
            for (int j = 0; j < CW; ++j) otile[tile_index<SWAP, BN>(row, cbeg + c0 + j)] = v[j];
          } else {                             // row pitch BN+4: 16-byte stores
#pragma unroll
            for (int j = 0; j < CW; j += 4)
              *reinterpret_cast<uint4*>(otile + tile_index<SWAP, BN>(row, cbeg + c0 + j)) =
                  make_uint4(v[j], v[j + 1], v[j + 2], v[j + 3]);
          }
        }
      }
      named_bar_sync(1, ET);
      if (epi_ok) write_out(0, 128, 0, BN);
    } else if (cluster_red && C::kPush) {
      // ---- cluster split-K, push: every thread stores its row of this
      // partial straight from registers into the owning CTA's receive slot
      // `kz` with asynchronous stores that count their bytes on that CTA's
      // barrier; each CTA waits for the bytes of the rows it owns and sums
      // them, in split order, into the output tile.  Only real outputs cross
      // the cluster: token columns < M under Swap-AB (decode tiles are mostly
      // padding), token rows < M otherwise.
      const int Sk = prm.split_k;
      const int owner = row / rows_per, rl = row % rows_per;
      const int cvalid = SWAP ? min(BN, Mlim - q0) : BN;
      const bool rvalid = SWAP || (p0 + row < prm.M);
      if (etid == 0) {
        // bytes this CTA receives: from each of the Sk CTAs, its owned rows
        // (Swap-AB: all rows_per; standard: those below M) x cvalid words
        const int r_own = (int)cluster_ctarank() * rows_per;
        const int rows_in = SWAP ? rows_per : max(0, min(rows_per, prm.M - p0 - r_own));
        mbar_arrive_expect_tx(recv_full, (uint32_t)(Sk * rows_in * cvalid * 4));
      }
      if (!epi_phase1) cluster_wait();         // phase 1: every receiver is initialised
      const uint32_t dst = mapa_shared(smem_u32(smem + L.recv) + (uint32_t)kz * slot_bytes, (uint32_t)owner);
      const uint32_t rbar = mapa_shared(smem_u32(recv_full), (uint32_t)owner);
#pragma unroll
      for (int c0 = 0; c0 < NC; c0 += CW) {
        if (cbeg + c0 >= cvalid) break;
        uint32_t v[CW];
        if (epi_ok) {
          load_chunk(c0, v);
        } else {
#pragma unroll
          for (int j = 0; j < CW; ++j) v[j] = 0u;
        }
        if (SWAP) {                            // slice [c][rl]: one word per lane, lanes contiguous
#pragma unroll
          for (int j = 0; j < CW; ++j)
            if (cbeg + c0 + j < cvalid)
              st_async_b32(dst + 4u * (uint32_t)slice_index<SWAP, BN>(rl, cbeg + c0 + j, rows_per), v[j], rbar);
        } else if (rvalid) {                   // slice [rl][c]: 16 bytes per store
#pragma unroll
          for (int j = 0; j < CW; j += 4)
            st_async_v4(dst + 4u * (uint32_t)slice_index<SWAP, BN>(rl, cbeg + c0 + j, rows_per), v[j], v[j + 1],
                        v[j + 2], v[j + 3], rbar);
        }
      }
      if (etid == 0) trace_at(prm, kTrSent);
      const bool got = __all_sync(0xffffffffu, mbar_wait_cluster(recv_full, 0, prm.err, prm.wait_ns));
      if (etid == 0) trace_at(prm, kTrRecv);
      const int r0 = (int)cluster_ctarank() * rows_per;
      const int zstride = rows_per * prm.recv_cols;
      // The owner reduces and stores in one pass: a slot keeps 8 consecutive
      // output channels contiguous (Swap-AB: per token column, the owned
      // channels; standard: per owned token row, the tile's channels), so a
      // unit of 8 channels is two 16-byte loads per split, summed in split
      // order, scaled and stored to y as one 16-byte vector (no output tile,
      // no barrier before the stores).
      if (epi_ok && got) {
        const uint32_t recv_s = smem_u32(smem + L.recv);
        const int nrow = SWAP ? cvalid : max(0, min(rows_per, prm.M - p0 - r0));   // slice rows with outputs
        const int ub = (SWAP ? rows_per : BN) / 8;                                // units per slice row
#pragma unroll 1
        for (int u = etid; u < nrow * ub; u += ET) {
          const int i = u / ub, j8 = (u - i * ub) * 8;
          // Swap-AB: i = token column, j8 = first owned channel; standard:
          // i = owned token row, j8 = first channel of the tile
          const int r = SWAP ? r0 + j8 : r0 + i;
          const int c = SWAP ? i : j8;
          const int m = SWAP ? q0 + i : p0 + r0 + i;
          const int n0 = SWAP ? p0 + r0 + j8 : q0 + j8;
          if (m >= Mlim || n0 >= prm.N) continue;
          uint32_t acc8[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
          // four splits' two 16-byte loads at a time, then their sums in split order
          const uint32_t a0 = recv_s + 4u * (uint32_t)(i * (SWAP ? rows_per : BN) + j8);
#pragma unroll
          for (int z0 = 0; z0 < kMaxClusterSplit; z0 += 4) {
            if (z0 >= Sk) break;
            uint4 wz[4][2];
#pragma unroll
            for (int dz = 0; dz < 4; ++dz) {
              if (z0 + dz < Sk) {
                const uint32_t a = a0 + 4u * (uint32_t)((z0 + dz) * zstride);
                wz[dz][0] = lds_v4(a);
                wz[dz][1] = lds_v4(a + 16u);
              }
            }
#pragma unroll
            for (int dz = 0; dz < 4; ++dz) {
              if (z0 + dz < Sk) {
                const uint32_t w[8] = {wz[dz][0].x, wz[dz][0].y, wz[dz][0].z, wz[dz][0].w,
                                       wz[dz][1].x, wz[dz][1].y, wz[dz][1].z, wz[dz][1].w};
#pragma unroll
                for (int k = 0; k < 8; ++k) acc8[k] = add_acc<FMT>(acc8[k], w[k]);
              }
            }
          }
          store8(r, c, m, n0, acc8);
        }
      }
      if (etid == 0) trace_at(prm, kTrReduced);
    } else if (cluster_red) {
      // ---- cluster split-K, pull: stage the partial in the idle ring; the
      // reduction runs after the cluster barrier below
      if (epi_ok) {
#pragma unroll
        for (int c0 = 0; c0 < NC; c0 += CW) {
          uint32_t v[CW];
          load_chunk(c0, v);
          if constexpr (SWAP) {
#pragma unroll
            for (int j = 0; j < CW; ++j) stage_buf[red_index<SWAP, BN>(row, cbeg + c0 + j)] = v[j];
          } else {
#pragma unroll
            for (int j = 0; j < CW; j += 4)
              *reinterpret_cast<uint4*>(stage_buf + red_index<SWAP, BN>(row, cbeg + c0 + j)) =
                  make_uint4(v[j], v[j + 1], v[j + 2], v[j + 3]);
          }
        }
      }
    } else if (epi_ok) {
      // ---- workspace split-K: partial to global memory
#pragma unroll
      for (int c0 = 0; c0 < NC; c0 += CW) {
        uint32_t v[CW];
        load_chunk(c0, v);
        if (prow_ok) {
#pragma unroll
          for (int j = 0; j < CW; ++j) {
            const int c = cbeg + c0 + j;
            const int m = SWAP ? q0 + c : prow;
            const int n = SWAP ? prow : q0 + c;
            if (m < Mlim && n < prm.N) part[(size_t)kz * MN + (size_t)m * prm.N + n] = v[j];
          }
        }
      }
      if (prm.reduce_mode == kReduceLastCta) {
        // Last-arriving CTA of this output tile sums the partials in split
        // order (deterministic) and applies the epilogue.
        __threadfence();
        named_bar_sync(1, ET);
        const unsigned tile = blockIdx.y * gridDim.x + blockIdx.x;
        if (etid == 0) {
          const unsigned prev = atomicAdd(&prm.counters[tile], 1u);
          *flag_last = (prev == (unsigned)(prm.split_k - 1));
        }
        named_bar_sync(1, ET);
        if (*flag_last) {
          __threadfence();
          if (prow_ok) {
            // 16 columns at a time: all their loads of one split are issued
            // before any store, so the L2 round trips overlap.
#pragma unroll 1
            for (int c0 = 0; c0 < NC; c0 += 16) {
              uint32_t acc[16];
#pragma unroll
              for (int j = 0; j < 16; ++j) acc[j] = 0u;
              // two splits per round: 32 loads in flight, summed in split order
              for (int z0 = 0; z0 < prm.split_k; z0 += 2) {
                uint32_t t[2][16];
#pragma unroll
                for (int dz = 0; dz < 2; ++dz) {
#pragma unroll
                  for (int j = 0; j < 16; ++j) {
                    const int c = cbeg + c0 + j;
                    const int m = SWAP ? q0 + c : prow;
                    const int n = SWAP ? prow : q0 + c;
                    t[dz][j] = (z0 + dz < prm.split_k && m < Mlim && n < prm.N)
                                   ? ld_u32_cg(part + (z0 + dz) * MN + (size_t)m * prm.N + n)
                                   : 0u;
                  }
                }
#pragma unroll
                for (int dz = 0; dz < 2; ++dz)
#pragma unroll
                  for (int j = 0; j < 16; ++j)
                    if (z0 + dz < prm.split_k) acc[j] = add_acc<FMT>(acc[j], t[dz][j]);
              }
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const int c = cbeg + c0 + j;
                const int m = SWAP ? q0 + c : prow;
                const int n = SWAP ? prow : q0 + c;
                if (m < Mlim && n < prm.N) emit<FMT, SWAP>(prm, row, c, m, n, acc[j], alpha, row_s, col_s);
              }
            }
          }
          if (etid == 0) prm.counters[tile] = 0u;
        }
      }
    }
  }

  // ------------------------------------------------ cluster barrier phases
  // Phase 1 was arrived at after set-up; push-mode epilogue warps have
  // already waited on it.  Pull mode adds phase 2 (every partial staged) and
  // phase 3 (every remote read done) around the reduction.
  if (cluster_red) {
    __syncwarp();
    if (!(warp >= 2 && (C::kPush || epi_phase1))) cluster_wait();
    if constexpr (!C::kPush) {
      cluster_sync();
      if (warp >= 2 && *flag_epi == 0) {
        const int etid = threadIdx.x - 64;
        const int Sk = prm.split_k;
        const uint32_t rank = cluster_ctarank();
        const int r0 = (int)rank * rows_per;
        const uint32_t red_s = smem_u32(smem + L.p);
        const float alpha = alpha_of<FMT>(prm, expert);
        // units of 8 consecutive output channels: 2 x 16-byte remote loads per
        // split, summed in split order, scaled and stored as one 16-byte vector.
        // Up to four splits: a thread's next unit's loads are in flight with
        // this unit's (two units per round), so one remote round trip serves two.
        const int units = rows_per * BN / 8;
        const bool vec = (prm.ldy % 8) == 0;
        auto unit_pos = [&](int u, int& r, int& c) {
          if (SWAP) { c = u / (rows_per / 8); r = r0 + (u % (rows_per / 8)) * 8; }
          else      { r = r0 + u / (BN / 8); c = (u % (BN / 8)) * 8; }
        };
        auto finish_unit = [&](int r, int c, const uint32_t (&acc8)[8]) {
          const int m = SWAP ? q0 + c : p0 + r;
          const int n0 = SWAP ? p0 + r : q0 + c;
          if (m >= Mlim || n0 >= prm.N) return;
          if (prm.out_kind == 1) {
            uint32_t* Yu = reinterpret_cast<uint32_t*>(prm.Y) + (size_t)m * prm.ldy;
            for (int j = 0; j < 8 && n0 + j < prm.N; ++j) Yu[n0 + j] = acc8[j];
            return;
          }
          float y8[8];
          float sa = 1.f, sw[8] = {1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f};
          if constexpr (FMT == kFP8 || FMT == kINT8) scales8<SWAP>(row_s, col_s, r, c, sa, sw);
#pragma unroll
          for (int j = 0; j < 8; ++j) y8[j] = finish_value<FMT>(acc8[j], sa, sw[j], alpha);
          __nv_bfloat16* Yb = reinterpret_cast<__nv_bfloat16*>(prm.Y) + (size_t)m * prm.ldy;
          if (vec && n0 + 8 <= prm.N) {
            uint32_t pk[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const __nv_bfloat162 b2 = __floats2bfloat162_rn(y8[2 * h], y8[2 * h + 1]);
              pk[h] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            *reinterpret_cast<uint4*>(Yb + n0) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          } else {
            for (int j = 0; j < 8 && n0 + j < prm.N; ++j) Yb[n0 + j] = __float2bfloat16_rn(y8[j]);
          }
        };
        if (Sk <= 4) {
          constexpr int kZ = 4;
#pragma unroll 1
          for (int u = etid; u < units; u += 2 * C::kEpiThreads) {
            const int u2 = u + C::kEpiThreads;
            int r[2], c[2];
            unit_pos(u, r[0], c[0]);
            unit_pos(u2 < units ? u2 : u, r[1], c[1]);
            uint4 t[2][kZ][2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint32_t off = 4u * (uint32_t)red_index<SWAP, BN>(r[h], c[h]);
#pragma unroll
              for (int z = 0; z < kZ; ++z) {
                if (z < Sk) {
                  t[h][z][0] = ld_dsmem_v4(mapa_shared(red_s + off, (uint32_t)z));
                  t[h][z][1] = ld_dsmem_v4(mapa_shared(red_s + off + 16u, (uint32_t)z));
                }
              }
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              if (h == 1 && u2 >= units) break;
              uint32_t acc8[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
              for (int z = 0; z < kZ; ++z) {
                if (z < Sk) {
                  const uint32_t w[8] = {t[h][z][0].x, t[h][z][0].y, t[h][z][0].z, t[h][z][0].w,
                                         t[h][z][1].x, t[h][z][1].y, t[h][z][1].z, t[h][z][1].w};
#pragma unroll
                  for (int j = 0; j < 8; ++j) acc8[j] = add_acc<FMT>(acc8[j], w[j]);
                }
              }
              finish_unit(r[h], c[h], acc8);
            }
          }
        } else {
#pragma unroll 1
          for (int u = etid; u < units; u += C::kEpiThreads) {
            int r, c;
            unit_pos(u, r, c);
            const uint32_t off = 4u * (uint32_t)red_index<SWAP, BN>(r, c);
            uint4 t[kMaxClusterSplit][2];
#pragma unroll
            for (int z = 0; z < kMaxClusterSplit; ++z) {
              if (z < Sk) {
                t[z][0] = ld_dsmem_v4(mapa_shared(red_s + off, (uint32_t)z));
                t[z][1] = ld_dsmem_v4(mapa_shared(red_s + off + 16u, (uint32_t)z));
              }
            }
            uint32_t acc8[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
            for (int z = 0; z < kMaxClusterSplit; ++z) {
              if (z < Sk) {
                const uint32_t w[8] = {t[z][0].x, t[z][0].y, t[z][0].z, t[z][0].w,
                                       t[z][1].x, t[z][1].y, t[z][1].z, t[z][1].w};
#pragma unroll
                for (int j = 0; j < 8; ++j) acc8[j] = add_acc<FMT>(acc8[j], w[j]);
              }
            }
            finish_unit(r, c, acc8);
          }
        }
      }
      __syncwarp();
      cluster_sync();
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) trace_at(prm, kTrDone);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemAlloc);
  }
}

// Second-pass split-K reduction: y[m, n] = epilogue(sum_z partial[z, m, n]),
// summed in split order.
template <int FMT>
__global__ void splitk_reduce_kernel(const GemmParams prm) {
  griddep_wait();
  griddep_launch_dependents();
  const size_t MN = (size_t)prm.M * prm.N;
  const uint32_t* part = reinterpret_cast<const uint32_t*>(prm.partial);
  for (size_t o = blockIdx.x * (size_t)blockDim.x + threadIdx.x; o < MN;
       o += (size_t)gridDim.x * blockDim.x) {
    const int m = (int)(o / prm.N), n = (int)(o % prm.N);
    uint32_t bits;
    if constexpr (FMT == kINT8) {
      int s = 0;
      for (int z = 0; z < prm.split_k; ++z) s += (int)__ldcg(part + z * MN + o);
      bits = (uint32_t)s;
    } else {
      float s = 0.f;
      for (int z = 0; z < prm.split_k; ++z) s += __uint_as_float(__ldcg(part + z * MN + o));
      bits = __float_as_uint(s);
    }
    if (prm.out_kind == 1) {
      reinterpret_cast<uint32_t*>(prm.Y)[(size_t)m * prm.ldy + n] = bits;
    } else {
      // grouped: row m belongs to the last expert whose first token is <= m
      // (offsets clamped to [0, M] as in the GEMM kernel)
      int expert = 0;
      if (prm.expert_offsets != nullptr) {
        int lo = 0, hi = prm.experts - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (min(max(__ldg(prm.expert_offsets + mid), 0), prm.M) <= m) lo = mid;
          else hi = mid - 1;
        }
        expert = lo;
      }
      float sa = 1.f, sw = 1.f;
      if constexpr (FMT == kFP8 || FMT == kINT8) {
        sa = __ldg(prm.scale_a + m);
        sw = __ldg(prm.scale_w + (size_t)expert * prm.N + n);
      }
      reinterpret_cast<__nv_bfloat16*>(prm.Y)[(size_t)m * prm.ldy + n] =
          __float2bfloat16_rn(finish_value<FMT>(bits, sa, sw, alpha_of<FMT>(prm, expert)));
    }
  }
}

}  // namespace qg
