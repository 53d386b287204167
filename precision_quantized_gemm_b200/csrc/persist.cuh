// persist.cuh — the persistent variant of the quantized GEMM for large M
// (qg_config.variant = 2): standard orientation, FP8_Dynamic and W8A8_INT8
// (qgemm_persist_kernel) and Block_FP8 (qgemm_persist_block_kernel, below).
//
// Why a third kernel: the tile kernel runs one 128 x BN output tile per CTA,
// so every tile pays the CTA's set-up, the pipeline fill and its epilogue
// with the tensor core idle (per-CTA stamps at M = 4096, N = K = 5120,
// 128 x 256 tiles: 13 us of mainloop, then 2.8 us of epilogue and ~1.3 us
// before the next CTA's first MMA).  Here one CTA per SM walks the tiles
// t = blockIdx.x, blockIdx.x + gridDim.x, ...; its producer streams the K
// tiles of consecutive tiles through one continuous ring, and TMEM holds two
// BN-column accumulators, so the MMAs of tile j + 1 run while the epilogue
// warps drain tile j (TMEM -> fp32 scales -> bf16 -> 128-byte-swizzled
// boxes -> TMA store through a tensor map of y).
//
// Roles: warp 0 producer (one thread), warp 1 MMA issuer (one thread; also
// allocates TMEM), warps 2-5 the epilogue (thread = TMEM lane = output row).
// Barriers: full / empty per ring slot, acc_full / acc_empty per accumulator.
// Every wait is bounded; a wait that gives up sets the abort word, and every
// role stops at its next check.  The MMAs of one tile accumulate their K
// tiles in the same order as the tile kernel's, and the epilogue applies the
// same fp32 arithmetic, so y is bitwise that of the tile kernel with the
// same tile_n.
#pragma once
#include "gemm_kernel.cuh"

namespace qg {

template <int FMT, int BN>
struct PsCfg {
  static constexpr int kThreads = 192;             // producer, MMA, 4 epilogue warps
  static constexpr int kQTileBytes = BN * kKTileBytes;
  static constexpr int kStage = kPTileBytes + kQTileBytes;
  // the bf16 output goes out in slices of up to 128 channels (two boxes of
  // 64), one slice buffer: a 256-wide tile leaves room for a 4-stage ring
  static constexpr int kYCols = BN < 128 ? BN : 128;
  static constexpr int kYBytes = 128 * kYCols * 2;
  static constexpr int kTmemCols = 2 * BN;         // two accumulators
  static constexpr uint32_t kIdesc = (FMT == kINT8) ? idesc_i8(BN) : idesc_f8f6f4_e4m3(BN);
  static_assert(FMT == kFP8 || FMT == kINT8, "persistent kernel: FP8_Dynamic and W8A8_INT8");
  static_assert(BN == 128 || BN == 256, "persistent kernel: 128- or 256-wide tiles");
};

// Shared memory: the ring (P tiles, then Q tiles), the y boxes, the channel
// scales of the tile, the barriers and the TMEM address / abort words
// (+ alignment slack).
struct PsLayout {
  uint32_t p, q, y, cols, bars, misc, total;
};
template <int FMT, int BN>
__host__ __device__ __forceinline__ PsLayout ps_layout(int stages) {
  using C = PsCfg<FMT, BN>;
  PsLayout L;
  L.p = 0;
  L.q = L.p + (uint32_t)stages * kPTileBytes;
  L.y = L.q + (uint32_t)stages * C::kQTileBytes;
  L.cols = L.y + C::kYBytes;
  L.bars = L.cols + 4u * BN;
  L.misc = L.bars + 8u * (2u * stages + 4u);
  L.total = L.misc + 16u;
  return L;
}
template <int FMT, int BN>
__host__ __device__ constexpr size_t ps_smem_bytes(int stages) {
  return (size_t)ps_layout<FMT, BN>(stages).total + 1024;
}

template <int FMT, int BN>
__global__ void __launch_bounds__(PsCfg<FMT, BN>::kThreads, 1)
    qgemm_persist_kernel(const __grid_constant__ CUtensorMap tmap_p, const __grid_constant__ CUtensorMap tmap_q,
                         const __grid_constant__ CUtensorMap tmap_y, const GemmParams prm) {
  using C = PsCfg<FMT, BN>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = prm.stages;
  const PsLayout L = ps_layout<FMT, BN>(S);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;              // [2]
  uint64_t* acc_empty = acc_full + 2;          // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc);
  volatile int* flag_abort = reinterpret_cast<volatile int*>(smem + L.misc + 4);
  float* col_s = reinterpret_cast<float*>(smem + L.cols);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // tiles: m-tile fastest, so the CTAs of one wave share weight tiles
  const int tp = (prm.M + 127) / 128, tq = (prm.N + BN - 1) / BN;
  const int tiles = tp * tq;
  const int nkt = prm.kt_total;

  if (threadIdx.x == 0) {
    prefetch_tmap(&tmap_p);
    prefetch_tmap(&tmap_q);
    prefetch_tmap(&tmap_y);
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);             // one arrival per epilogue warp
    }
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
  if (threadIdx.x == 0) {
    trace_at(prm, kTrReady);
    griddep_launch_dependents();
  }

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // both operands are re-read by other tiles of the wave: keep them in L2
      const uint64_t pol = policy_evict_last();
      griddep_wait();                          // the activations come from the preceding kernel
      bool ok = true;
      int issued = 0;                          // K tiles issued over all of this CTA's tiles
      int st = 0, r = 0;                       // slot of the next K tile, and its round
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        const int p0 = (t % tp) * 128, q0 = (t / tp) * BN;
        for (int kt = 0; kt < nkt; ++kt) {
          // the slot's previous round must have been consumed by the MMAs
          if (r > 0 && !mbar_wait(&empty[st], (uint32_t)((r - 1) & 1), prm.err, prm.wait_ns)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[st], C::kStage);
          tma_load_2d(smem + L.p + (size_t)st * kPTileBytes, &tmap_p, &full[st], kt * kKTileBytes, p0, pol);
          tma_load_2d(smem + L.q + (size_t)st * C::kQTileBytes, &tmap_q, &full[st], kt * kKTileBytes, q0, pol);
          ++issued;
          if (++st == S) { st = 0; ++r; }
        }
        if (*flag_abort) ok = false;
      }
      if (!ok) {
        *flag_abort = 1;
        // drain: wait (bounded) until every issued copy has landed
        for (int g = (issued > S ? issued - S : 0); g < issued; ++g)
          mbar_wait(&full[g % S], (uint32_t)((g / S) & 1), prm.err, prm.wait_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint64_t dp0 = sdesc_sw128(smem_u32(smem + L.p));
      const uint64_t dq0 = sdesc_sw128(smem_u32(smem + L.q));
      int st = 0;
      uint32_t ph = 0;
      bool ok = true;
      int j = 0;                               // this CTA's tile count; accumulator j & 1
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++j) {
        const int ab = j & 1;
        // the epilogue has read tile j - 2 out of this accumulator
        if (j >= 2 && !mbar_wait(&acc_empty[ab], (uint32_t)(((j >> 1) - 1) & 1), prm.err, prm.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_t = tmem_base + (uint32_t)(ab * BN);
        for (int kt = 0; kt < nkt; ++kt) {
          if (!mbar_wait(&full[st], ph, prm.err, prm.wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint64_t dp = dp0 + (uint64_t)((st * kPTileBytes) >> 4);
          const uint64_t dq = dq0 + (uint64_t)((st * C::kQTileBytes) >> 4);
#pragma unroll
          for (int s = 0; s < 4; ++s) {        // 32 bytes of K per MMA
            const uint32_t accum = (kt > 0 || s > 0);
            if constexpr (FMT == kINT8) mma_i8(d_t, dp + (uint64_t)(2 * s), dq + (uint64_t)(2 * s), C::kIdesc, accum);
            else mma_f8f6f4(d_t, dp + (uint64_t)(2 * s), dq + (uint64_t)(2 * s), C::kIdesc, accum);
          }
          mma_commit(&empty[st]);
          if (++st == S) { st = 0; ph ^= 1u; }
        }
        if (!ok) break;
        mma_commit(&acc_full[ab]);
        if (*flag_abort) ok = false;
      }
      if (!ok) *flag_abort = 1;
    }
  } else {
    // --------------------------------------------------------------- epilogue
    const int quarter = warp & 3;              // TMEM lanes this warp may access
    const int row = quarter * 32 + lane;       // output row of the tile
    const int etid = threadIdx.x - 64;         // 0 .. 127
    const uint32_t lane_addr = tmem_base + ((uint32_t)(quarter * 32) << 16);
    uint8_t* ybuf = smem + L.y;
    griddep_wait();                            // the activation scales come from the preceding kernel
    const float alpha = alpha_of<FMT>(prm);
    int j = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++j) {
      const int ab = j & 1;
      const int p0 = (t % tp) * 128, q0 = (t / tp) * BN;
      // the tile's channel scales, and the previous tile's boxes read out by its store
      for (int c = etid; c < BN; c += 128) col_s[c] = (q0 + c < prm.N) ? __ldg(prm.scale_w + q0 + c) : 0.f;
      if (etid == 0) bulk_wait_read_all();
      const bool got = mbar_wait(&acc_full[ab], (uint32_t)((j >> 1) & 1), prm.err, prm.wait_ns);
      if (!__all_sync(0xffffffffu, got)) *flag_abort = 1;
      // scales staged, boxes free; every epilogue warp takes the same abort decision
      if (named_bar_or(1, 128, *flag_abort != 0)) break;
      tc_fence_after();
      const float sa = (p0 + row < prm.M) ? __ldg(prm.scale_a + p0 + row) : 0.f;
#pragma unroll
      for (int y0 = 0; y0 < BN; y0 += C::kYCols) {   // slices of the tile's channels
        if (y0 > 0) {                          // the previous slice's boxes read out by its store
          if (etid == 0) bulk_wait_read_all();
          named_bar_sync(1, 128);
        }
#pragma unroll
        for (int c0 = y0; c0 < y0 + C::kYCols; c0 += 32) {
          uint32_t v[32];
          tmem_ld32(lane_addr + (uint32_t)(ab * BN + c0), v);
          tmem_ld_wait();
          if (c0 + 32 == BN) {                 // the accumulator is in registers: free it for tile j + 2
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[ab]);
          }
#pragma unroll
          for (int k = 0; k < 32; k += 8) {
            const int col = c0 + k;            // a multiple of 8
            const float4 s0 = reinterpret_cast<const float4*>(col_s + col)[0];
            const float4 s1 = reinterpret_cast<const float4*>(col_s + col)[1];
            const float sw[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
            uint32_t pk[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const __nv_bfloat162 b2 =
                  __floats2bfloat162_rn(finish_value<FMT>(v[k + 2 * h], sa, sw[2 * h], alpha),
                                        finish_value<FMT>(v[k + 2 * h + 1], sa, sw[2 * h + 1], alpha));
              pk[h] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            // 16-byte chunk (col % 64) / 8 of row `row` of the slice's box, 128-byte swizzle
            const int lc = col - y0;
            const uint32_t off = (uint32_t)(lc >> 6) * 16384u + (uint32_t)row * 128u +
                                 ((uint32_t)(((lc & 63) >> 3) ^ (row & 7)) << 4);
            *reinterpret_cast<uint4*>(ybuf + off) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (etid == 0) {
#pragma unroll
          for (int b = 0; b < C::kYCols / 64; ++b)
            tma_store_2d(&tmap_y, ybuf + b * 16384, (q0 + y0 + b * 64) * 2, p0);
          bulk_commit();
        }
      }
    }
    if (etid == 0) {
      bulk_wait_all();                         // every store performed before the CTA ends
      trace_at(prm, kTrDone);
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ---------------------------------------------------------------- Block_FP8
// The persistent kernel for Block_FP8: the same tile walk and continuous
// ring, with the tile kernel's promotion (Cfg<kBLOCK, BN>: every 128-K group
// lands in one of kNAcc TMEM buffers, the epilogue warps fold it into fp32
// register accumulators, acc += p_g * (s_a * s_w), with fma.rn.f32x2).  The
// group buffers are free as soon as a tile's last group is promoted, so the
// MMAs of tile j + 1 start while the epilogue warps round and store tile j
// from registers.  The group counter and the buffers' phases run on over
// the tiles; the scales of each tile are staged in shared memory after the
// previous tile's promotion has read its own.
struct PbLayout {
  uint32_t p, q, y, sa, sw, bars, misc, total;
};
template <int BN>
__host__ __device__ __forceinline__ PbLayout pb_layout(int stages, int nkt) {
  PbLayout L;
  L.p = 0;
  L.q = L.p + (uint32_t)stages * kPTileBytes;
  L.y = L.q + (uint32_t)stages * (BN * kKTileBytes);
  L.sa = L.y + 128u * 128u * 2u;               // one 128-channel slice of bf16 output
  L.sw = L.sa + 4u * 128u * (uint32_t)nkt;     // activation scales [row][group]
  L.bars = (L.sw + 4u * (BN / 128) * (uint32_t)nkt + 7u) & ~7u;   // weight scales [group][block]
  L.misc = L.bars + 8u * (2u * stages + 2u * Cfg<kBLOCK, BN>::kNAcc);
  L.total = L.misc + 16u;
  return L;
}
template <int BN>
__host__ __device__ constexpr size_t pb_smem_bytes(int stages, int nkt) {
  return (size_t)pb_layout<BN>(stages, nkt).total + 1024;
}

// Threads: a role warpgroup (warp 0 producer, warp 1 MMA issuer, warps 2-3
// idle) and the promotion warps (Cfg<kBLOCK, BN>::kEpiWarps).  With 16
// promotion warps (BN = 256) each thread keeps 64 promoted columns; the role
// warpgroup gives registers to the promotion warpgroups by setmaxnreg.
template <int BN>
struct PbCfg {
  static constexpr int kEpiWarps = Cfg<kBLOCK, BN>::kEpiWarps;
  static constexpr int kThreads = 128 + 32 * kEpiWarps;
  static constexpr bool kRegSplit = kEpiWarps >= 16;
  // 640 threads launch with 96 registers (five warps per SM sub-partition);
  // 128 x 40 + 512 x 104 <= 640 x 96
  static constexpr int kRegsLaunch = 96, kRegsRole = 40, kRegsEpi = 104;
  static_assert(!kRegSplit || (kThreads == 640 && 128 * kRegsRole + 512 * kRegsEpi <= 640 * kRegsLaunch),
                "register split beyond the launch allocation");
};

template <int BN>
__global__ void __launch_bounds__(PbCfg<BN>::kThreads, 1)
    qgemm_persist_block_kernel(const __grid_constant__ CUtensorMap tmap_p, const __grid_constant__ CUtensorMap tmap_q,
                               const __grid_constant__ CUtensorMap tmap_y, const GemmParams prm) {
  using C = Cfg<kBLOCK, BN>;
  static_assert(BN == 128 || BN == 256, "persistent Block_FP8: 128- or 256-wide tiles");
  constexpr int ET = C::kEpiThreads;
  constexpr int NC = C::kCols;                 // promoted columns per epilogue thread
  constexpr int NA = C::kNAcc;                 // TMEM group buffers
  constexpr int WB = BN / 128;                 // 128-row weight blocks per tile
  constexpr int kTmemCols = NA * BN;           // 512
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = prm.stages;
  const int nkt = prm.kt_total;                // K tiles = 128-wide groups
  const int G = prm.groups;
  const PbLayout L = pb_layout<BN>(S, nkt);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;                 // [NA]
  uint64_t* tempty = tfull + NA;               // [NA]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc);
  volatile int* flag_abort = reinterpret_cast<volatile int*>(smem + L.misc + 4);
  float* sa_s = reinterpret_cast<float*>(smem + L.sa);
  float* sw_s = reinterpret_cast<float*>(smem + L.sw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tp = (prm.M + 127) / 128, tq = (prm.N + BN - 1) / BN;
  const int tiles = tp * tq;

  if (threadIdx.x == 0) {
    prefetch_tmap(&tmap_p);
    prefetch_tmap(&tmap_q);
    prefetch_tmap(&tmap_y);
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < NA; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], C::kEpiWarps);
    }
    *flag_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  if (threadIdx.x == 0) {
    trace_at(prm, kTrReady);
    griddep_launch_dependents();
  }

  using PC = PbCfg<BN>;
  if (warp < 4) {
  // the role warpgroup; its setmaxnreg opens the branch so that it governs
  // the code after it
  if constexpr (PC::kRegSplit) reg_release<PC::kRegsRole>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      griddep_wait();
      bool ok = true;
      int issued = 0, st = 0, r = 0;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        const int p0 = (t % tp) * 128, q0 = (t / tp) * BN;
        for (int kt = 0; kt < nkt; ++kt) {
          if (r > 0 && !mbar_wait(&empty[st], (uint32_t)((r - 1) & 1), prm.err, prm.wait_ns)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[st], kPTileBytes + BN * kKTileBytes);
          tma_load_2d(smem + L.p + (size_t)st * kPTileBytes, &tmap_p, &full[st], kt * kKTileBytes, p0, pol);
          tma_load_2d(smem + L.q + (size_t)st * (BN * kKTileBytes), &tmap_q, &full[st], kt * kKTileBytes, q0, pol);
          ++issued;
          if (++st == S) { st = 0; ++r; }
        }
        if (*flag_abort) ok = false;
      }
      if (!ok) {
        *flag_abort = 1;
        for (int g = (issued > S ? issued - S : 0); g < issued; ++g)
          mbar_wait(&full[g % S], (uint32_t)((g / S) & 1), prm.err, prm.wait_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint64_t dp0 = sdesc_sw128(smem_u32(smem + L.p));
      const uint64_t dq0 = sdesc_sw128(smem_u32(smem + L.q));
      int st = 0, gb = 0, gr = 0;              // ring slot; group buffer and its round (over all tiles)
      uint32_t ph = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        for (int kt = 0; kt < nkt; ++kt) {
          if (!mbar_wait(&full[st], ph, prm.err, prm.wait_ns)) { ok = false; break; }
          if (gr > 0 && !mbar_wait(&tempty[gb], (uint32_t)((gr - 1) & 1), prm.err, prm.wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint64_t dp = dp0 + (uint64_t)((st * kPTileBytes) >> 4);
          const uint64_t dq = dq0 + (uint64_t)((st * (BN * kKTileBytes)) >> 4);
          const uint32_t d_t = tmem_base + (uint32_t)(gb * BN);
#pragma unroll
          for (int s = 0; s < 4; ++s)          // one 128-K group per K tile: a fresh sum
            mma_f8f6f4(d_t, dp + (uint64_t)(2 * s), dq + (uint64_t)(2 * s), C::kIdesc, s > 0 ? 1u : 0u);
          mma_commit(&empty[st]);
          mma_commit(&tfull[gb]);
          if (++gb == NA) { gb = 0; ++gr; }
          if (++st == S) { st = 0; ph ^= 1u; }
        }
        if (*flag_abort) ok = false;
      }
      if (!ok) *flag_abort = 1;
    }
  }
  } else {
    if constexpr (PC::kRegSplit) reg_acquire<PC::kRegsEpi>();
    // ------------------------------------------------ promotion and epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int etid = threadIdx.x - 128;
    const int cbeg = ((warp - 4) / 4) * NC;    // this thread's columns [cbeg, cbeg + NC)
    const uint32_t lane_addr = tmem_base + ((uint32_t)(quarter * 32) << 16);
    uint8_t* ybuf = smem + L.y;
    griddep_wait();                            // the activation scales come from the preceding kernel
    const int nblk = (prm.N + 127) / 128;
    int gb = 0, gr = 0;                        // group buffer and its round, as the MMA issuer counts
    for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
      const int p0 = (t % tp) * 128, q0 = (t / tp) * BN;
      // this tile's scales (the previous tile's promotion is done with its own)
      for (int idx = etid; idx < 128 * nkt; idx += ET) {
        const int rr = idx / nkt, gl = idx % nkt;
        const int m = p0 + rr;
        sa_s[idx] = (m < prm.M) ? __ldg(prm.scale_a + (size_t)m * G + gl) : 0.f;
      }
      for (int idx = etid; idx < WB * nkt; idx += ET) {
        const int gl = idx / WB, jb = idx % WB;
        const int b = q0 / 128 + jb;
        sw_s[idx] = (b < nblk) ? __ldg(prm.scale_w + (size_t)b * G + gl) : 0.f;
      }
      if (named_bar_or(1, ET, *flag_abort != 0)) break;
      uint64_t acc2[NC / 2];
#pragma unroll
      for (int c = 0; c < NC / 2; ++c) acc2[c] = 0ull;
      bool ok = true;
      for (int i = 0; i < nkt; ++i) {
        ok = __all_sync(0xffffffffu, mbar_wait(&tfull[gb], (uint32_t)(gr & 1), prm.err, prm.wait_ns));
        if (!ok) break;
        tc_fence_after();
        const float f_row = sa_s[row * nkt + i];
        constexpr int PB = C::kEpiWarps >= 16 ? 16 : 32;   // columns per TMEM load
        constexpr int NCH = NC / PB;
        auto ld_chunk = [&](int c0, uint32_t (&v)[PB]) {
          if constexpr (PB == 32) tmem_ld32(lane_addr + (uint32_t)(gb * BN + cbeg + c0), v);
          else tmem_ld16(lane_addr + (uint32_t)(gb * BN + cbeg + c0), v);
        };
        auto fma_chunk = [&](int c0, const uint32_t (&v)[PB]) {
          // one weight block per chunk (chunks never cross a 128-column block)
          const float f = f_row * sw_s[i * WB + (WB == 2 ? (cbeg + c0) / 128 : 0)];
          const uint64_t f2 = pack_f32x2(f, f);
#pragma unroll
          for (int j = 0; j < PB; j += 2) ffma2(acc2[(c0 + j) / 2], v[j], v[j + 1], f2);
        };
        // the next chunk's TMEM load is in flight while this chunk's FMAs run
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
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[gb]);
        if (++gb == NA) { gb = 0; ++gr; }
      }
      if (!ok) *flag_abort = 1;
      // the promoted sums rounded to bf16 pairs: half the registers through
      // the store phase
      uint32_t yb[NC / 2];
#pragma unroll
      for (int c = 0; c < NC / 2; ++c) {
        uint32_t lo, hi;
        unpack_u32x2(acc2[c], lo, hi);
        const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(lo), __uint_as_float(hi));
        yb[c] = *reinterpret_cast<const uint32_t*>(&b2);
      }
      // every warp's promotion done (or given up); one abort decision for all
      if (named_bar_or(1, ET, *flag_abort != 0)) break;
      // ---- store from registers, one 128-channel slice at a time
#pragma unroll
      for (int y0 = 0; y0 < BN; y0 += 128) {
        if (etid == 0) bulk_wait_read_all();   // the previous slice's boxes read out by its store
        named_bar_sync(1, ET);
        if (cbeg >= y0 && cbeg < y0 + 128) {
#pragma unroll
          for (int c = 0; c < NC; c += 8) {
            const int lc = cbeg + c - y0;      // channel within the slice, a multiple of 8
            const uint32_t off = (uint32_t)(lc >> 6) * 16384u + (uint32_t)row * 128u +
                                 ((uint32_t)(((lc & 63) >> 3) ^ (row & 7)) << 4);
            *reinterpret_cast<uint4*>(ybuf + off) =
                make_uint4(yb[c / 2], yb[c / 2 + 1], yb[c / 2 + 2], yb[c / 2 + 3]);
          }
        }
        fence_proxy_async_smem();
        named_bar_sync(1, ET);
        if (etid == 0) {
          tma_store_2d(&tmap_y, ybuf, (q0 + y0) * 2, p0);
          tma_store_2d(&tmap_y, ybuf + 16384, (q0 + y0 + 64) * 2, p0);
          bulk_commit();
        }
      }
    }
    if (etid == 0) {
      bulk_wait_all();
      trace_at(prm, kTrDone);
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace qg
