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
// Warp roles (192 threads):
//   warp 0      TMA producer: weights first (they do not depend on the
//               preceding kernel), then griddepcontrol.wait, then activations;
//               a `stages`-deep ring of 128-byte K tiles in shared memory.
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer.
//   warps 2..5  epilogue: tcgen05.ld of the fp32/int32 accumulator, scales in
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
// in a workspace that the last-arriving CTA or a second kernel sums.  Every
// mode adds the partials in split order, so results are deterministic and
// identical across modes.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "ptx.cuh"

namespace qg {

enum Fmt : int { kFP8 = 0, kINT8 = 1, kBLOCK = 2, kNVF4 = 3 };

constexpr int kKTileBytes = 128;     // bytes of K per pipeline stage (one 128B swizzle row)
constexpr int kPTileBytes = 128 * kKTileBytes;
constexpr int kSfAtomBytes = 512;    // one 128x4 atom of e4m3 block scales

constexpr int kReduceCluster = 0;    // split-K partials summed through distributed shared memory
constexpr int kReduceSecondPass = 1; // partials in the workspace, summed by a second kernel
constexpr int kReduceLastCta = 2;    // partials in the workspace, summed by the last-arriving CTA
constexpr int kMaxClusterSplit = 8;

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
  unsigned long long* trace;   // optional: kTraceEvents timestamps per CTA (ns)
  int nkt_max;                 // most K tiles any split slice holds: ceil(kt_total / split_k)
  int recv_cols;               // cluster push: token columns per receive slot (0: no receive buffer)
};

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
  kTrSpare = 11,
  kTraceEvents = 12
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
  static constexpr int kNAcc = kBlock ? (BN >= 256 ? 2 : 4) : 1;  // TMEM accumulators
  // Wide Block_FP8 tiles promote with 8 epilogue warps: two per 32-lane TMEM
  // quarter, each owning half of the columns.
  static constexpr int kEpiWarps = (kBlock && BN >= 128) ? 8 : 4;
  static constexpr int kEpiThreads = 32 * kEpiWarps;
  static constexpr int kThreads = 64 + kEpiThreads;
  static constexpr int kCols = BN / (kEpiWarps / 4);               // columns per epilogue thread
  // CTAs per SM the register budget must allow: narrow (decode) tiles keep
  // room for the next launch's CTAs to start streaming weights early.
  static constexpr int kMinBlocks = (!kBlock && BN <= 64) ? 3 : (kBlock && BN <= 32) ? 2 : 1;
  static constexpr int kSfaCol = kNAcc * BN;                       // TMEM column of SF A
  static constexpr int kSfbCol = kSfaCol + 16;                     // 4 steps x 4 words
  static constexpr int kTmemUsed = kNvf4 ? kSfbCol + 16 * kSfQAtoms : kNAcc * BN;
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
  uint32_t p, q, sfp, sfq, recv, bars, misc, epis, scales, total;
};
template <int FMT, bool SWAP, int BN>
__host__ __device__ inline SmemLayout smem_layout(int stages, int nkt_max, int recv_cols) {
  using C = Cfg<FMT, BN>;
  SmemLayout L;
  L.p = 0;
  L.q = L.p + stages * kPTileBytes;
  L.sfp = L.q + stages * C::kQTileBytes;
  L.sfq = L.sfp + stages * C::kSfPBytes;
  L.recv = L.sfq + stages * C::kSfQBytes;
  L.bars = L.recv + (C::kPush ? 4u * 128u * (uint32_t)recv_cols : 0u);
  // full[stages], empty[stages], acc_full, tfull[4], tempty[4], recv_full
  L.misc = L.bars + 8 * (2 * stages + 1 + 8 + 1);
  L.epis = (L.misc + 16 + 15) & ~15u;          // row / column scales (FP8, INT8)
  L.scales = L.epis + (C::kRowColScales ? 4 * (128 + BN) : 0);
  L.total = L.scales + (C::kBlock ? 4u * (uint32_t)((block_act_rows<SWAP, BN>() +
                                                     block_weight_blocks<SWAP, BN>()) * nkt_max)
                                  : 0u);
  return L;
}
template <int FMT, bool SWAP, int BN>
__host__ inline size_t smem_bytes(int stages, int nkt_max, int recv_cols) {
  return smem_layout<FMT, SWAP, BN>(stages, nkt_max, recv_cols).total + 1024;  // + alignment slack
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

template <int FMT>
__device__ __forceinline__ float alpha_of(const GemmParams& prm) {
  if constexpr (FMT == kNVF4) return __ldg(prm.g_a) * __ldg(prm.g_w);
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

template <int FMT, bool SWAP, int BN>
__global__ void __launch_bounds__(Cfg<FMT, BN>::kThreads, Cfg<FMT, BN>::kMinBlocks)
    qgemm_kernel(const __grid_constant__ CUtensorMap tmap_p,
                 const __grid_constant__ CUtensorMap tmap_q, const GemmParams prm) {
  using C = Cfg<FMT, BN>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const SmemLayout L = smem_layout<FMT, SWAP, BN>(prm.stages, prm.nkt_max, prm.recv_cols);
  const int S = prm.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;
  uint64_t* tfull = acc_full + 1;
  uint64_t* tempty = tfull + 4;
  uint64_t* recv_full = tempty + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc);
  volatile int* flag_last = reinterpret_cast<volatile int*>(smem + L.misc + 4);
  volatile int* flag_abort = reinterpret_cast<volatile int*>(smem + L.misc + 8);
  volatile int* flag_epi = reinterpret_cast<volatile int*>(smem + L.misc + 12);
  float* row_s = reinterpret_cast<float*>(smem + L.epis);
  float* col_s = row_s + 128;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int p0 = blockIdx.x * 128;
  const int q0 = blockIdx.y * BN;
  const int kz = blockIdx.z;
  const int kt_begin = (int)(((long long)kz * prm.kt_total) / prm.split_k);
  const int kt_end = (int)(((long long)(kz + 1) * prm.kt_total) / prm.split_k);
  const int nkt = kt_end - kt_begin;
  if (threadIdx.x == 0) trace_at(prm, kTrEntry);
  const bool cluster_red = prm.split_k > 1 && prm.reduce_mode == kReduceCluster;
  const int rows_per = 128 / prm.split_k;                  // cluster mode: rows owned per CTA
  const uint32_t slot_bytes = 4u * (uint32_t)(rows_per * prm.recv_cols);

  if (threadIdx.x == 0) {
    prefetch_tmap(&tmap_p);
    prefetch_tmap(&tmap_q);
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(acc_full, 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], C::kEpiWarps);
    }
    // push mode: each of the 128 rows of the owned slices arrives once, from
    // whichever CTA computed it (split_k CTAs x 128/split_k rows)
    mbar_init(recv_full, 128);
    *flag_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
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
      const int row_w = SWAP ? p0 : q0;
      const int row_a = SWAP ? q0 : p0;
      // NVFP4 scale atoms: P rows [p0, p0+128) are one 128-row block; Q has
      // one or two blocks (the second only if it holds any row).
      const int sfq_atoms = (C::kSfQAtoms == 2 && q0 + 128 < prm.rows_q) ? 2 : 1;
      const uint32_t stage_tx = kPTileBytes + C::kQTileBytes +
                                (C::kNvf4 ? (uint32_t)(4 * kSfAtomBytes * (1 + sfq_atoms)) : 0u);
      auto load_w = [&](int i) {
        const int st = i % S;
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
      auto load_a = [&](int i) {
        const int st = i % S;
        const int kt = kt_begin + i;
        tma_load_2d(smem + off_a + st * bytes_a, map_a, &full[st], kt * kKTileBytes, row_a, pol_a);
        if constexpr (C::kNvf4) {
          const uint8_t* sfa = SWAP ? prm.sf_q : prm.sf_p;
          const int rb = row_a / 128;
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
        load_w(i);
        if (i == 0) trace_at(prm, kTrFirstLoad);
      }
      griddep_wait();
      trace_at(prm, kTrDepWait);
      for (int i = 0; i < pre; ++i) load_a(i);
      bool ok = true;
      int issued = pre;
      for (int i = pre; i < nkt; ++i) {
        const int st = i % S;
        if (!mbar_wait(&empty[st], ((i / S) - 1) & 1, prm.err)) { ok = false; break; }
        mbar_arrive_expect_tx(&full[st], stage_tx);
        load_w(i);
        load_a(i);
        issued = i + 1;
      }
      if (!ok) {
        *flag_abort = 1;
        // Drain: wait (bounded) until every issued copy has landed.
        for (int i = (issued > S ? issued - S : 0); i < issued; ++i)
          mbar_wait(&full[i % S], (i / S) & 1, prm.err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0 && nkt > 0) {
      const uint32_t sp = smem_u32(smem + L.p);
      const uint32_t sq = smem_u32(smem + L.q);
      const uint32_t ssfp = smem_u32(smem + L.sfp);
      const uint32_t ssfq = smem_u32(smem + L.sfq);
      const uint32_t sfa_t = tmem_base + C::kSfaCol;
      const uint32_t sfb_t = tmem_base + C::kSfbCol;
      // word offset of this CTA's first Q row inside its 128-row SF atom
      const uint32_t sfb_word = (uint32_t)((q0 % 128) / 32);
      for (int i = 0; i < nkt; ++i) {
        const int st = i % S;
        if (*flag_abort || !mbar_wait(&full[st], (i / S) & 1, prm.err)) { *flag_abort = 1; break; }
        if (i == 0) trace_at(prm, kTrFirstFull);
        uint32_t d_t = tmem_base;
        if constexpr (C::kBlock) {
          const int b = i % C::kNAcc;
          const int r = i / C::kNAcc;
          if (r > 0 && !mbar_wait(&tempty[b], (r - 1) & 1, prm.err)) { *flag_abort = 1; break; }
          d_t = tmem_base + b * BN;
        }
        tc_fence_after();
        if constexpr (C::kNvf4) {
          for (int s = 0; s < 4; ++s) {
            tmem_cp_32x128b_x4(sfa_t + 4 * s,
                               sdesc_plain_32x16(ssfp + st * C::kSfPBytes + s * kSfAtomBytes));
            for (int a = 0; a < C::kSfQAtoms; ++a)
              tmem_cp_32x128b_x4(sfb_t + 4 * C::kSfQAtoms * s + 4 * a,
                                 sdesc_plain_32x16(ssfq + st * C::kSfQBytes + a * 4 * kSfAtomBytes +
                                                   s * kSfAtomBytes));
          }
        }
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint64_t da = sdesc_sw128(sp + st * kPTileBytes + 32 * s);
          const uint64_t db = sdesc_sw128(sq + st * C::kQTileBytes + 32 * s);
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
        if constexpr (C::kBlock) mma_commit(&tfull[i % C::kNAcc]);
      }
      if constexpr (!C::kBlock) mma_commit(acc_full);
      trace_at(prm, kTrLastMma);
    }
  } else {
    // --------------------------------------------------------------- epilogue
    constexpr int EW = C::kEpiWarps;
    constexpr int ET = C::kEpiThreads;
    constexpr int NC = C::kCols;
    constexpr int CW = NC >= 32 ? 32 : NC;     // accumulator columns per TMEM load
    const int quarter = warp & 3;              // TMEM lanes this warp may access
    const int row = quarter * 32 + lane;       // row of P in the tile
    const int etid = threadIdx.x - 64;         // 0..ET-1
    const int cbeg = ((warp - 2) / 4) * NC;    // this thread's columns [cbeg, cbeg + NC)
    const uint32_t lane_addr = tmem_base + ((uint32_t)(quarter * 32) << 16);
    griddep_wait();                            // scales/partials of earlier kernels
    // FP8 / INT8: stage the per-row scales of this tile while the mainloop runs
    if constexpr (C::kRowColScales) {
      const float* sp = SWAP ? prm.scale_w : prm.scale_a;
      const float* sq = SWAP ? prm.scale_a : prm.scale_w;
      for (int r = etid; r < 128; r += ET) row_s[r] = (p0 + r < prm.rows_p) ? __ldg(sp + p0 + r) : 0.f;
      for (int c = etid; c < BN; c += ET) col_s[c] = (q0 + c < prm.rows_q) ? __ldg(sq + q0 + c) : 0.f;
    }
    bool ok = true;                            // warp-uniform
    float acc_f[NC];                           // Block_FP8 promoted accumulator
    if constexpr (C::kBlock) {
      float* sa_s = reinterpret_cast<float*>(smem + L.scales);          // act scales
      constexpr int act_rows = block_act_rows<SWAP, BN>();
      float* sw_s = sa_s + act_rows * prm.nkt_max;                      // weight scales
      const int G = prm.groups;
      const int g0 = kt_begin;
      // Stage this CTA's scales: activations per (row, group), weights per
      // (128-row block, group).
      const int act_base = SWAP ? q0 : p0;
      for (int idx = etid; idx < act_rows * nkt; idx += ET) {
        const int r = idx / nkt, gl = idx % nkt;
        const int m = act_base + r;
        sa_s[idx] = (m < prm.M) ? __ldg(prm.scale_a + (size_t)m * G + g0 + gl) : 0.f;
      }
      constexpr int WB = block_weight_blocks<SWAP, BN>();              // weight blocks per tile
      const int wrow0 = (SWAP ? p0 : q0) / 128;
      const int nblk = (prm.N + 127) / 128;
      for (int idx = etid; idx < WB * nkt; idx += ET) {
        const int gl = idx / WB, jb = idx % WB;
        const int b = wrow0 + jb;
        sw_s[idx] = (b < nblk) ? __ldg(prm.scale_w + (size_t)b * G + g0 + gl) : 0.f;
      }
      named_bar_sync(1, ET);
#pragma unroll
      for (int c = 0; c < NC; ++c) acc_f[c] = 0.f;
      for (int i = 0; i < nkt; ++i) {
        const int b = i % C::kNAcc;
        ok = __all_sync(0xffffffffu, mbar_wait(&tfull[b], (i / C::kNAcc) & 1, prm.err));
        if (!ok) break;
        tc_fence_after();
        // acc += p_g * (s_a * s_w): one FMA per element
        float f_row = 0.f;
        if (!SWAP) f_row = sa_s[row * nkt + i];
        // columns per TMEM round trip: 64 (two loads, one wait) while the
        // accumulator is small, 32 when it already holds 128 registers
        constexpr int PB = NC >= 128 ? 32 : 64;
#pragma unroll
        for (int c0 = 0; c0 < NC; c0 += PB) {
          uint32_t v[PB];
          if constexpr (NC % 32 == 0) {
            tmem_ld32(lane_addr + b * BN + cbeg + c0, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
            if constexpr (PB == 64)
              if (c0 + 32 < NC)
                tmem_ld32(lane_addr + b * BN + cbeg + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
          } else {                             // 16-column tiles: stay inside the buffer
            tmem_ld16(lane_addr + b * BN + cbeg + c0, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
          }
          tmem_ld_wait();
          if (SWAP) {
            const float sw = sw_s[i];
#pragma unroll
            for (int j = 0; j < PB && c0 + j < NC; ++j)
              acc_f[c0 + j] = fmaf(__uint_as_float(v[j]), sa_s[(cbeg + c0 + j) * nkt + i] * sw, acc_f[c0 + j]);
          } else {
#pragma unroll
            for (int j = 0; j < PB && c0 + j < NC; ++j) {
              const float f = f_row * sw_s[i * WB + (WB == 2 ? (cbeg + c0 + j) / 128 : 0)];
              acc_f[c0 + j] = fmaf(__uint_as_float(v[j]), f, acc_f[c0 + j]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[b]);
      }
    } else {
      ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0, prm.err));
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
    const float alpha = alpha_of<FMT>(prm);
    // Accumulator columns [cbeg + c0, cbeg + c0 + CW) of this thread's row.
    auto load_chunk = [&](int c0, uint32_t (&v)[CW]) {
      if constexpr (C::kBlock) {
#pragma unroll
        for (int j = 0; j < CW; ++j) v[j] = __float_as_uint(acc_f[c0 + j]);
      } else if constexpr (CW == 32) {
        tmem_ld32(lane_addr + cbeg + c0, v);
        tmem_ld_wait();
      } else {
        tmem_ld16(lane_addr + cbeg + c0, v);
        tmem_ld_wait();
      }
    };

    // Output tile in the idle ring: raw accumulator bits of tile element
    // (r, c) at otile[tile_index(r, c)], written out by one compact loop that
    // scales, converts and stores 16-byte vectors along the contiguous
    // dimension of y (channels: r under Swap-AB, c otherwise).
    uint32_t* otile = stage_buf;
    auto write_out = [&](int r_begin, int r_count, int c_begin, int c_count) {
      const int units = SWAP ? c_count * (r_count / 8) : r_count * (c_count / 8);
      const bool vec = (prm.ldy % 8) == 0;
#pragma unroll 1
      for (int u = etid; u < units; u += ET) {
        int r, c;                              // first of 8 consecutive output channels
        if (SWAP) { c = c_begin + u / (r_count / 8); r = r_begin + (u % (r_count / 8)) * 8; }
        else      { r = r_begin + u / (c_count / 8); c = c_begin + (u % (c_count / 8)) * 8; }
        const int m = SWAP ? q0 + c : p0 + r;
        const int n0 = SWAP ? p0 + r : q0 + c;
        if (m >= prm.M || n0 >= prm.N) continue;
        const uint4* src = reinterpret_cast<const uint4*>(otile + tile_index<SWAP, BN>(r, c));
        const uint4 w0 = src[0], w1 = src[1];
        const uint32_t acc8[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        if (prm.out_kind == 1) {
          uint32_t* Yu = reinterpret_cast<uint32_t*>(prm.Y) + (size_t)m * prm.ldy;
          for (int j = 0; j < 8 && n0 + j < prm.N; ++j) Yu[n0 + j] = acc8[j];
          continue;
        }
        float y8[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float sa = 1.f, sw = 1.f;
          if constexpr (FMT == kFP8 || FMT == kINT8) {
            sa = SWAP ? col_s[c] : row_s[r];
            sw = SWAP ? row_s[r + j] : col_s[c + j];
          }
          y8[j] = finish_value<FMT>(acc8[j], sa, sw, alpha);
        }
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
      }
    };

    if (!split) {
      // ---- direct: accumulator -> tile -> y
      if (epi_ok) {
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
      // `kz` and arrives (release) on that CTA's barrier; each CTA sums the
      // rows it owns, in split order, into the output tile.  Only real
      // outputs cross the cluster: token columns < M under Swap-AB (decode
      // tiles are mostly padding), token rows < M otherwise.
      const int Sk = prm.split_k;
      const int owner = row / rows_per, rl = row % rows_per;
      const int cvalid = SWAP ? min(BN, prm.M - q0) : BN;
      const bool rvalid = SWAP || (p0 + row < prm.M);
      cluster_wait();                          // phase 1: every receiver is initialised
      const uint32_t dst = mapa_shared(smem_u32(smem + L.recv) + (uint32_t)kz * slot_bytes, (uint32_t)owner);
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
              st_dsmem_b32(dst + 4u * (uint32_t)slice_index<SWAP, BN>(rl, cbeg + c0 + j, rows_per), v[j]);
        } else if (rvalid) {                   // slice [rl][c]: 16 bytes per store
#pragma unroll
          for (int j = 0; j < CW; j += 4)
            st_dsmem_v4(dst + 4u * (uint32_t)slice_index<SWAP, BN>(rl, cbeg + c0 + j, rows_per), v[j], v[j + 1],
                        v[j + 2], v[j + 3]);
        }
      }
      mbar_arrive_remote(mapa_shared(smem_u32(recv_full), (uint32_t)owner));
      if (etid == 0) trace_at(prm, kTrSent);
      const bool got = __all_sync(0xffffffffu, mbar_wait_cluster(recv_full, 0, prm.err));
      if (etid == 0) trace_at(prm, kTrRecv);
      const uint32_t* __restrict__ recv = reinterpret_cast<const uint32_t*>(smem + L.recv);
      uint32_t* __restrict__ ot = otile;
      const int r0 = (int)cluster_ctarank() * rows_per;
      const int zstride = rows_per * prm.recv_cols;
      if (epi_ok && got) {
        // fixed per-thread row (Swap-AB) or column (standard), stepping over
        // the other index: no divisions in the loop, loads of later
        // iterations overlap
        if (SWAP) {
          const int rl2 = etid % rows_per, cstep = ET / rows_per;
          const uint32_t recv_s = smem_u32(smem + L.recv);
#pragma unroll 4
          for (int c = etid / rows_per; c < cvalid; c += cstep) {
            uint32_t acc = 0u;
            for (int z = 0; z < Sk; ++z)
              acc = add_acc<FMT>(acc, lds_u32(recv_s + 4u * (uint32_t)(z * zstride + c * rows_per + rl2)));
            ot[tile_index<SWAP, BN>(r0 + rl2, c)] = acc;
          }
        } else {
          const int nrow = max(0, min(rows_per, prm.M - p0 - r0));
          const int c = etid % BN, rstep = ET / BN;
#pragma unroll 4
          for (int rl2 = etid / BN; rl2 < nrow; rl2 += rstep) {
            uint32_t acc = 0u;
            for (int z = 0; z < Sk; ++z) acc = add_acc<FMT>(acc, recv[z * zstride + rl2 * BN + c]);
            ot[tile_index<SWAP, BN>(r0 + rl2, c)] = acc;
          }
        }
      }
      named_bar_sync(1, ET);
      if (etid == 0) trace_at(prm, kTrReduced);
      if (epi_ok && got) write_out(r0, rows_per, 0, BN);
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
            if (m < prm.M && n < prm.N) part[(size_t)kz * MN + (size_t)m * prm.N + n] = v[j];
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
                    t[dz][j] = (z0 + dz < prm.split_k && m < prm.M && n < prm.N)
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
                if (m < prm.M && n < prm.N) emit<FMT, SWAP>(prm, row, c, m, n, acc[j], alpha, row_s, col_s);
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
    if (!(C::kPush && warp >= 2)) cluster_wait();
    if constexpr (!C::kPush) {
      cluster_sync();
      if (warp >= 2 && *flag_epi == 0) {
        const int etid = threadIdx.x - 64;
        const int Sk = prm.split_k;
        const uint32_t rank = cluster_ctarank();
        const int r0 = (int)rank * rows_per;
        const uint32_t red_s = smem_u32(smem + L.p);
        const float alpha = alpha_of<FMT>(prm);
        // units of 8 consecutive output channels: 2 x 16-byte remote loads per
        // split, summed in split order, scaled and stored as one 16-byte vector
        const int units = rows_per * BN / 8;
        const bool vec = (prm.ldy % 8) == 0;
#pragma unroll 1
        for (int u = etid; u < units; u += C::kEpiThreads) {
          int r, c;
          if (SWAP) { c = u / (rows_per / 8); r = r0 + (u % (rows_per / 8)) * 8; }
          else      { r = r0 + u / (BN / 8); c = (u % (BN / 8)) * 8; }
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
          const int m = SWAP ? q0 + c : p0 + r;
          const int n0 = SWAP ? p0 + r : q0 + c;
          if (m >= prm.M || n0 >= prm.N) continue;
          if (prm.out_kind == 1) {
            uint32_t* Yu = reinterpret_cast<uint32_t*>(prm.Y) + (size_t)m * prm.ldy;
            for (int j = 0; j < 8 && n0 + j < prm.N; ++j) Yu[n0 + j] = acc8[j];
            continue;
          }
          float y8[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float sa = 1.f, sw = 1.f;
            if constexpr (FMT == kFP8 || FMT == kINT8) {
              sa = SWAP ? col_s[c] : row_s[r];
              sw = SWAP ? row_s[r + j] : col_s[c + j];
            }
            y8[j] = finish_value<FMT>(acc8[j], sa, sw, alpha);
          }
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
    tmem_dealloc(tmem_base, C::kTmemCols);
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
  float alpha = 1.f;
  if constexpr (FMT == kNVF4) alpha = __ldg(prm.g_a) * __ldg(prm.g_w);
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
      float sa = 1.f, sw = 1.f;
      if constexpr (FMT == kFP8 || FMT == kINT8) {
        sa = __ldg(prm.scale_a + m);
        sw = __ldg(prm.scale_w + n);
      }
      reinterpret_cast<__nv_bfloat16*>(prm.Y)[(size_t)m * prm.ldy + n] =
          __float2bfloat16_rn(finish_value<FMT>(bits, sa, sw, alpha));
    }
  }
}

}  // namespace qg
