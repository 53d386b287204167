// pair.cuh — Block_FP8 on CTA pairs (qg_config.variant = 3): standard
// orientation, output tiles of 256 tokens x BN (128 or 256) channels, each
// computed by the two CTAs of a cluster with one cta_group::2 MMA per
// 32-byte K step.
//
// Why: Block_FP8's promotion folds every 128-K group's partial sum into fp32
// registers, so the MMAs of group g + NA wait until the promotion of group g
// has freed its TMEM buffer.  A CTA holds 512 TMEM columns: two buffers for
// a 256-channel tile, four for a 128-channel one, but a 128 x 128 tile
// streams 1.31x the operand bytes per output of a 128 x 256 tile.  A pair
// tile of 256 x 128 has the operand bytes per output of 128 x 256 (each CTA
// loads its 128 token rows and half of the 128 weight rows) and the four
// 128-column buffers of a 128-channel tile, so four groups are in flight
// between an MMA and the promotion that frees its buffer.  The issuing
// thread spends ~600 cycles per group on four pair MMAs and their two
// commits, more than the ~360 cycles of tensor work of a 256 x 128 group,
// so 256 x 256 pair tiles (two 256-column buffers) double the work per
// issued MMA.
//
// Roles: warp 0 of each CTA loads its own operand halves; their bytes
// complete on the even CTA's ring barrier.  Warp 1 of each CTA allocates the
// pair's TMEM; warp 1 of the even CTA issues the MMAs (M = 256) and commits
// them to the ring and group barriers of both CTAs (warps 0-3, the role
// warpgroup, run on 40 registers).  Warps 4-19 of each CTA (104 registers)
// promote their own 128 TMEM lanes (= token rows), acc += p_g * (s_a * s_w)
// with fma.rn.f32x2 as the tile kernel does, and arrive on the even CTA's
// buffer-free barrier.  The pairs walk the tiles persistently (tile t =
// pair, pair + pairs, ...); the rounded output leaves through TMA stores.
// Every wait is bounded; a wait that gives up sets the abort word and the
// device error, and both CTAs meet at the cluster barrier before exiting.
#pragma once
#include "gemm_kernel.cuh"

namespace qg {

template <int BN>
struct PpCfg {
  static_assert(BN == 128 || BN == 256, "CTA pairs: 256 x 128 or 256 x 256 tiles");
  static constexpr int kBN = BN;                   // channels per pair tile
  static constexpr int kBHalf = kBN / 2;           // weight rows each CTA loads
  static constexpr int kEpiWarps = 16;             // four per TMEM lane quarter
  static constexpr int kThreads = 128 + 32 * kEpiWarps;
  // 640 threads launch with 96 registers; the role warpgroup gives its share
  // to the promotion warps (128 x 40 + 512 x 104 <= 640 x 96)
  static constexpr int kRegsLaunch = 96, kRegsRole = 40, kRegsEpi = 104;
  static_assert(128 * kRegsRole + 32 * kEpiWarps * kRegsEpi <= kThreads * kRegsLaunch,
                "register split beyond the launch allocation");
  static constexpr int kNC = kBN * 4 / kEpiWarps;  // promoted channels per thread
  static constexpr int kNAcc = 512 / kBN;          // TMEM group buffers
  static constexpr int kTmemCols = kNAcc * kBN;    // 512
  static constexpr int kQBytes = kBHalf * kKTileBytes;
  static constexpr int kStageBytes = kPTileBytes + kQBytes;   // per CTA
  static constexpr uint32_t kIdesc = idesc_f8f6f4_e4m3(kBN, 256);
  static constexpr int kPB = 16;                   // columns per TMEM load in the promotion
  static constexpr int kYCols = 128;               // output slice (two boxes of 64 channels)
};

// Shared memory per CTA: the ring (A tiles, then weight half tiles), one
// 128 x 128 bf16 output slice, the barriers, the TMEM address and abort
// words.  (The promotion reads its scales straight from global memory, two
// groups ahead.)
struct PpLayout {
  uint32_t p, q, y, bars, misc, total;
};
template <int BN>
__host__ __device__ __forceinline__ PpLayout pp_layout(int stages) {
  using P = PpCfg<BN>;
  PpLayout L;
  L.p = 0;
  L.q = L.p + (uint32_t)stages * kPTileBytes;
  L.y = L.q + (uint32_t)stages * P::kQBytes;
  L.bars = L.y + 128u * P::kYCols * 2u;
  L.misc = L.bars + 8u * (2u * stages + 2u * P::kNAcc);
  L.total = L.misc + 16u;
  return L;
}
template <int BN>
__host__ __device__ inline size_t pp_smem_bytes(int stages) {
  return (size_t)pp_layout<BN>(stages).total + 1024;
}

template <int BN>
__global__ void __launch_bounds__(PpCfg<BN>::kThreads, 1)
    qgemm_pair_block_kernel(const __grid_constant__ CUtensorMap tmap_p, const __grid_constant__ CUtensorMap tmap_q,
                            const __grid_constant__ CUtensorMap tmap_y, const GemmParams prm) {
  using P = PpCfg<BN>;
  constexpr int ET = 32 * P::kEpiWarps;
  constexpr int NC = P::kNC;
  constexpr int NA = P::kNAcc;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = prm.stages;
  const int nkt = prm.kt_total;                // K tiles = 128-wide groups
  const int G = prm.groups;
  const PpLayout L = pp_layout<BN>(S);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;                 // [NA]
  uint64_t* tempty = tfull + NA;               // [NA], used in the even CTA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc);
  volatile int* flag_abort = reinterpret_cast<volatile int*>(smem + L.misc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank() & 1u;            // 0: the pair's MMA issuer
  const uint32_t even = cluster_ctarank() & ~1u;
  const uint16_t pair_mask = (uint16_t)(3u << even);
  const int tp2 = (prm.M + 255) / 256, tq = (prm.N + P::kBN - 1) / P::kBN;
  const int tiles = tp2 * tq;
  const int pair = (int)(blockIdx.x >> 1), pairs = (int)(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    prefetch_tmap(&tmap_p);
    prefetch_tmap(&tmap_q);
    prefetch_tmap(&tmap_y);
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);                  // the even CTA's producer arrives (with both CTAs' bytes)
      mbar_init(&empty[i], 1);                 // the pair's MMA commit
    }
    for (int i = 0; i < NA; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 2 * P::kEpiWarps); // every promotion warp of both CTAs
    }
    *flag_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, P::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  cluster_sync();                              // both CTAs' barriers and TMEM exist
  if (threadIdx.x == 0) {
    trace_at(prm, kTrReady);
    griddep_launch_dependents();
  }

  if (warp < 4) {
  // the role warpgroup; its setmaxnreg opens the branch so that it governs
  // the code after it
  reg_release<P::kRegsRole>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      const uint32_t full_even = mapa_shared(smem_u32(&full[0]), even);
      griddep_wait();
      bool ok = true;
      int issued = 0, st = 0, r = 0;
      for (int t = pair; t < tiles && ok; t += pairs) {
        const int p0 = (t % tp2) * 256 + (int)rank * 128, q0 = (t / tp2) * P::kBN;
        for (int kt = 0; kt < nkt; ++kt) {
          if (r > 0 && !mbar_wait(&empty[st], (uint32_t)((r - 1) & 1), prm.err, prm.wait_ns)) { ok = false; break; }
          if (rank == 0) mbar_arrive_expect_tx(&full[st], 2u * P::kStageBytes);
          tma_load_2d_pair(smem + L.p + (size_t)st * kPTileBytes, &tmap_p, full_even + 8u * (uint32_t)st,
                           kt * kKTileBytes, p0, pol);
          tma_load_2d_pair(smem + L.q + (size_t)st * P::kQBytes, &tmap_q, full_even + 8u * (uint32_t)st,
                           kt * kKTileBytes, q0 + (int)rank * P::kBHalf, pol);
          ++issued;
          if (++st == S) { st = 0; ++r; }
        }
        if (*flag_abort) ok = false;
      }
      if (!ok) {
        *flag_abort = 1;
        // the even CTA's ring barriers count both CTAs' bytes: drain what
        // was issued before leaving (bounded)
        if (rank == 0)
          for (int g = (issued > S ? issued - S : 0); g < issued; ++g)
            mbar_wait(&full[g % S], (uint32_t)((g / S) & 1), prm.err, prm.wait_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer (even CTA)
    if (rank == 0 && lane == 0) {
      const uint64_t dp0 = sdesc_sw128(smem_u32(smem + L.p));
      const uint64_t dq0 = sdesc_sw128(smem_u32(smem + L.q));
      int st = 0, gb = 0, gr = 0;              // ring slot; group buffer and its round
      uint32_t ph = 0;
      bool ok = true;
      for (int t = pair; t < tiles && ok; t += pairs) {
        for (int kt = 0; kt < nkt; ++kt) {
          if (!mbar_wait(&full[st], ph, prm.err, prm.wait_ns)) { ok = false; break; }
          // the buffer's promotion in both CTAs is done (their TMEM loads
          // waited for and fenced before the arrivals)
          if (gr > 0 && !mbar_wait(&tempty[gb], (uint32_t)((gr - 1) & 1), prm.err, prm.wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint64_t dp = dp0 + (uint64_t)((st * kPTileBytes) >> 4);
          const uint64_t dq = dq0 + (uint64_t)((st * P::kQBytes) >> 4);
          const uint32_t d_t = tmem_base + (uint32_t)(gb * P::kBN);
#pragma unroll
          for (int s = 0; s < 4; ++s)          // one 128-K group per K tile: a fresh sum
            mma_f8f6f4_pair(d_t, dp + (uint64_t)(2 * s), dq + (uint64_t)(2 * s), P::kIdesc, s > 0 ? 1u : 0u);
          mma_commit_pair(&empty[st], pair_mask);
          mma_commit_pair(&tfull[gb], pair_mask);
          if (++gb == NA) { gb = 0; ++gr; }
          if (++st == S) { st = 0; ph ^= 1u; }
        }
        if (*flag_abort) ok = false;
      }
      if (!ok) *flag_abort = 1;
    }
  }
  } else {
    reg_acquire<P::kRegsEpi>();
    // ------------------------------------------------ promotion and epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int etid = threadIdx.x - 128;
    const int cbeg = ((warp - 4) / 4) * NC;    // this thread's channels [cbeg, cbeg + NC)
    const uint32_t lane_addr = tmem_base + ((uint32_t)(quarter * 32) << 16);
    const uint32_t tempty_even = mapa_shared(smem_u32(&tempty[0]), even);
    uint8_t* ybuf = smem + L.y;
    griddep_wait();                            // the activation scales come from the preceding kernel
    const int nblk = (prm.N + 127) / 128;
    int gb = 0, gr = 0;                        // group buffer and its round, as the MMA issuer counts
    for (int t = pair; t < tiles; t += pairs) {
      const int p0 = (t % tp2) * 256 + (int)rank * 128, q0 = (t / tp2) * P::kBN;
      if (named_bar_or(1, ET, *flag_abort != 0)) break;   // one abort decision for all warps
      // this row's activation scale and the tile's weight-block scale per
      // group, loaded two groups ahead of their use
      // this row's activation scale per group, loaded two groups ahead of
      // its use, and the weight-block scale of this thread's channels (its
      // NC channels lie in one 128-row weight block; one short row of
      // scales per block, read by every thread of the block: cached)
      const int m = p0 + row, bb = q0 / 128 + cbeg / 128;
      const bool live = m < prm.M && bb < nblk;
      const float* sa_g = prm.scale_a + (size_t)(live ? m : 0) * G;
      const float* sw_g = prm.scale_w + (size_t)(live ? bb : 0) * G;
      auto ld_sa = [&](int i) { return (live && i < nkt) ? __ldg(sa_g + i) : 0.f; };
      auto ld_sw = [&](int i) { return (live && i < nkt) ? __ldg(sw_g + i) : 0.f; };
      float sa0 = ld_sa(0), sa1 = ld_sa(1);
      uint64_t acc2[NC / 2];
#pragma unroll
      for (int c = 0; c < NC / 2; ++c) acc2[c] = 0ull;
      bool ok = true;
      constexpr int PB = P::kPB, NCH = NC / PB;
      for (int i = 0; i < nkt; ++i) {
        const float sa2 = ld_sa(i + 2);
        const float sw = ld_sw(i);
        ok = __all_sync(0xffffffffu, mbar_wait(&tfull[gb], (uint32_t)(gr & 1), prm.err, prm.wait_ns));
        if (!ok) break;
        tc_fence_after();
        const uint32_t base = lane_addr + (uint32_t)(gb * BN + cbeg);
        const float f = sa0 * sw;
        const uint64_t f2 = pack_f32x2(f, f);
        auto fma_chunk = [&](int c0, const uint32_t (&v)[PB]) {
#pragma unroll
          for (int j = 0; j < PB; j += 2) ffma2(acc2[(c0 + j) / 2], v[j], v[j + 1], f2);
        };
        // the next chunk's TMEM load is in flight while this chunk's FMAs run
        uint32_t va[PB], vb[PB];
        tmem_ld16(base, va);
        tmem_ld_wait();
#pragma unroll
        for (int ch = 0; ch < NCH; ch += 2) {
          if (ch + 1 < NCH) tmem_ld16(base + (uint32_t)((ch + 1) * PB), vb);
          fma_chunk(ch * PB, va);
          if (ch + 1 < NCH) {
            tmem_ld_wait();
            if (ch + 2 < NCH) tmem_ld16(base + (uint32_t)((ch + 2) * PB), va);
            fma_chunk((ch + 1) * PB, vb);
            if (ch + 2 < NCH) tmem_ld_wait();
          }
        }
        sa0 = sa1;
        sa1 = sa2;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(tempty_even + 8u * (uint32_t)gb);
        if (++gb == NA) { gb = 0; ++gr; }
      }
      if (!ok) *flag_abort = 1;
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
      // 128-channel slices (two boxes of 64: 128-byte rows, 128-byte swizzle)
      // through one buffer
#pragma unroll
      for (int y0 = 0; y0 < BN; y0 += P::kYCols) {
        if (etid == 0) bulk_wait_read_all();   // the previous slice's boxes read out by its store
        named_bar_sync(1, ET);
        if (cbeg >= y0 && cbeg < y0 + P::kYCols) {
#pragma unroll
          for (int c = 0; c < NC; c += 8) {
            const int lc = cbeg + c - y0;
            const uint32_t off = (uint32_t)(lc >> 6) * 16384u + (uint32_t)row * 128u +
                                 ((uint32_t)(((lc & 63) >> 3) ^ (row & 7)) << 4);
            *reinterpret_cast<uint4*>(ybuf + off) =
                make_uint4(yb[c / 2], yb[c / 2 + 1], yb[c / 2 + 2], yb[c / 2 + 3]);
          }
        }
        fence_proxy_async_smem();
        named_bar_sync(1, ET);
        // (the odd CTA's rows of the last pair tile may all lie beyond M: no
        // box starts outside y)
        if (etid == 0 && p0 < prm.M && q0 + y0 < prm.N) {
          tma_store_2d(&tmap_y, ybuf, (q0 + y0) * 2, p0);
          if (q0 + y0 + 64 < prm.N) tma_store_2d(&tmap_y, ybuf + 16384, (q0 + y0 + 64) * 2, p0);
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
  // The pair's MMAs into this CTA's TMEM and the peer's arrivals on this
  // CTA's barriers are done once both CTAs are here.
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, P::kTmemCols);
  }
}

}  // namespace qg
