// skinny.cuh — the decode ("skinny") variant of the quantized GEMM for a few
// tokens (M <= 32 per token tile): warp-level MMAs whose accumulators stay in
// registers, over a weight slice streamed into shared memory by TMA.
//
// Why a second kernel: at decode sizes the tile kernel (qgemm_kernel) is a
// latency chain, not a bandwidth one.  Per-CTA clocks of its Swap-AB launches
// show, after the weights and activations have arrived, ~490 cycles of the
// single issuing thread per 128-byte K tile (four tcgen05.mma of N = 16 and a
// commit), then the TMEM load, the split-K exchange through distributed shared
// memory and the owner's sum: 2 - 2.5 us of a 5.5 us INT8 4096^2 launch.
// Here every warp issues its own small MMAs in parallel and each CTA owns a
// few weight rows over the whole of K, so there is no split-K, no cross-CTA
// reduction and no tensor-memory round trip.
//
// Layout of the work.  CTA (x, y) computes y[m, n] for tokens m in
// [y*TM, y*TM + TM) and weight rows n in [x*R, x*R + R), R = 8*NF.  One
// producer warp streams K tiles (128 bytes of K) of the R weight rows and the
// TM token rows through a `stages`-deep ring: the weight tiles before the
// dependency wait, the activation tiles (written by the preceding kernel)
// after it.  Eight compute warps: warp w owns the 8 weight rows of n-fragment
// w % NF and the K tiles i with i % KG == w / NF (KG = 8 / NF), so every ring
// slot always feeds the same group of NF warps.  Per 32-byte K step a warp
// loads the token fragment (ldmatrix.x4 per 16 tokens) and the weight
// fragment (ldmatrix.x4 covers two K steps) from the 128-byte-swizzled tiles
// and issues mma.sync m16n8k32 (A = tokens, B = the weight rows).
// Block_FP8 promotes every K tile (one 128-K group) in registers:
// acc += p_g * (s_a * s_w).  The K groups of warps then meet in shared memory
// and are summed in K-group order (deterministic); the epilogue applies the
// scales in fp32 and stores bf16, 8 channels per 16-byte store.
#pragma once
#include <type_traits>

#include "gemm_kernel.cuh"

namespace qg {

// TM = 16 or 32: the tokens are the MMA's 16-row A operand and the weight
// rows its 8-column B operand (a warp owns 8 weight rows).  TM = 8 (up to 8
// tokens): the roles swap, the weight rows fill the 16-row A operand and the
// tokens the 8 columns (a warp owns 16 weight rows), which halves the MMAs
// per weight byte when a CTA has at most 8 tokens.
template <int FMT, int TM, int NF>
struct SkCfg {
  static constexpr bool kWA = TM == 8;           // weights as the A operand
  static constexpr int kR = 8 * NF;              // weight rows per CTA
  static constexpr int kUnits = kWA ? NF / 2 : NF;   // warps per K group
  static constexpr int kKG = 8 / kUnits;         // K groups of compute warps
  static constexpr int kWarps = 8;               // compute warps
  static constexpr int kThreads = 32 * (kWarps + 1);
  static constexpr int kMF = kWA ? 1 : TM / 16;  // A fragments per warp and K step
  static constexpr int kWTile = kR * kKTileBytes;
  static constexpr int kATile = TM * kKTileBytes;
  static constexpr int kStage = kWTile + kATile; // a multiple of 1024 (swizzle atoms)
  static constexpr int kRedBytes = kWarps * kMF * 16 * 8 * 4;
  static_assert(!kWA || NF >= 2, "weights as A need 16 rows per warp");
};

// Shared memory of a skinny launch: the ring, one full and one empty barrier
// per slot, the K-group reduction area (+ alignment slack).
template <int FMT, int TM, int NF>
__host__ __device__ constexpr size_t skinny_smem_bytes(int stages) {
  using C = SkCfg<FMT, TM, NF>;
  return (size_t)stages * C::kStage + 16u * (size_t)stages + (size_t)C::kRedBytes + 1024;
}

template <int FMT, int TM, int NF>
__global__ void __launch_bounds__(SkCfg<FMT, TM, NF>::kThreads, 1)
    qgemm_skinny_kernel(const __grid_constant__ CUtensorMap tmap_w,
                        const __grid_constant__ CUtensorMap tmap_a, const GemmParams prm) {
  using C = SkCfg<FMT, TM, NF>;
  constexpr bool kInt = FMT == kINT8;
  using Acc = typename std::conditional<kInt, int, float>::type;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = prm.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)S * C::kStage);
  uint64_t* empty = full + S;
  Acc* red = reinterpret_cast<Acc*>(empty + S);   // [warp][mf][16 tokens][8 rows]
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * C::kR;
  const int m0 = blockIdx.y * TM;
  const int nkt = prm.kt_total;
  bool ok = true;                              // this thread's waits all completed
  if (threadIdx.x == 0) trace_at(prm, kTrEntry);

  if (threadIdx.x == 0) {
    prefetch_tmap(&tmap_w);
    prefetch_tmap(&tmap_a);
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], C::kUnits);       // the warps of the slot's K group
    }
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    trace_at(prm, kTrReady);
    griddep_launch_dependents();
  }

  if (warp == C::kWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_a = policy_evict_last();
      const int pre = nkt < S ? nkt : S;
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(&full[i], C::kStage);
        tma_load_2d(smem + (size_t)i * C::kStage, &tmap_w, &full[i], i * kKTileBytes, n0, pol_w);
        if (i == 0) trace_at(prm, kTrFirstLoad);
      }
      if (prm.l2_ahead > 0) {
        // the weight rows of the CTA l2_ahead places later in launch order
        const long long t = (long long)blockIdx.x + (long long)gridDim.x * blockIdx.y + prm.l2_ahead;
        if (t < (long long)gridDim.x * gridDim.y) {
          const int tn0 = (int)(t % gridDim.x) * C::kR;
          for (int kt = 0; kt < nkt; ++kt) tma_prefetch_l2_2d(&tmap_w, kt * kKTileBytes, tn0);
        }
      }
      griddep_wait();                          // activations come from the preceding kernel
      trace_at(prm, kTrDepWait);
      for (int i = 0; i < pre; ++i)
        tma_load_2d(smem + (size_t)i * C::kStage + C::kWTile, &tmap_a, &full[i], i * kKTileBytes, m0, pol_a);
      int issued = pre;
      int st = 0;                              // slot of K tile i; parity of its previous use
      uint32_t ph = 0;
      for (int i = pre; i < nkt; ++i) {
        if (!mbar_wait(&empty[st], ph, prm.err, prm.wait_ns)) { ok = false; break; }
        mbar_arrive_expect_tx(&full[st], C::kStage);
        uint8_t* dst = smem + (size_t)st * C::kStage;
        tma_load_2d(dst, &tmap_w, &full[st], i * kKTileBytes, n0, pol_w);
        tma_load_2d(dst + C::kWTile, &tmap_a, &full[st], i * kKTileBytes, m0, pol_a);
        issued = i + 1;
        if (++st == S) { st = 0; ph ^= 1u; }
      }
      if (!ok) {
        // drain: wait (bounded) until every issued copy has landed
        for (int i = (issued > S ? issued - S : 0); i < issued; ++i)
          mbar_wait(&full[i % S], (i / S) & 1, prm.err, prm.wait_ns);
      }
    }
  } else {
    // ------------------------------------------------------- compute warps
    // weight rows [8 nf, 8 nf + 8) of the CTA (weights as A: [16 nf, 16 nf + 16))
    const int nf = warp % C::kUnits;
    const int kg = warp / C::kUnits;           // K tiles i with i % KG == kg
    const int g = lane >> 2, t = lane & 3;     // fragment row group and column pair
    // the activation scales below come from the preceding kernel
    griddep_wait();
    // one accumulator set per 32-byte K step of a tile, so that a warp's
    // MMAs do not wait on each other; summed in a fixed order at the end
    Acc acc[4][C::kMF][4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int mf = 0; mf < C::kMF; ++mf)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[q][mf][j] = (Acc)0;
    // ldmatrix row addresses (swizzled: the 16-byte chunk c of row r sits at
    // chunk c ^ (r % 8) of its 128-byte row)
    // B operand rows (8; two K steps per ldmatrix.x4): weight rows, or tokens
    const int brow = (C::kWA ? 0 : nf * 8) + (lane & 7);
    const int bchk = lane >> 3;                // chunk offset 0..3 (two K steps)
    // A operand rows (16 per fragment): tokens, or weight rows
    const int arow = (C::kWA ? nf * 16 : 0) + ((lane >> 3) & 1) * 8 + (lane & 7);
    const int achk = lane >> 4;                // chunk offset 0 / 1 (bytes 0-15 / 16-31 of a K step)
    const int G = prm.groups;
    for (int i = kg; i < nkt; i += C::kKG) {
      const int st = i % S;
      // Block_FP8: this group's scales, loaded while the tile may still be in flight
      float sw = 0.f, sa_lo[C::kMF], sa_hi[C::kMF];
      if constexpr (FMT == kBLOCK) {
        sw = __ldg(prm.scale_w + (size_t)(n0 / 128) * G + i);
#pragma unroll
        for (int mf = 0; mf < C::kMF; ++mf) {
          // the tokens of this thread's accumulator elements: rows g, g + 8 of
          // a 16-token fragment, or columns 2t, 2t + 1 (weights as A)
          const int mlo = C::kWA ? m0 + 2 * t : m0 + mf * 16 + g;
          const int mhi = C::kWA ? mlo + 1 : mlo + 8;
          sa_lo[mf] = (mlo < prm.M) ? __ldg(prm.scale_a + (size_t)mlo * G + i) : 0.f;
          sa_hi[mf] = (mhi < prm.M) ? __ldg(prm.scale_a + (size_t)mhi * G + i) : 0.f;
        }
      }
      if (!mbar_wait(&full[st], (uint32_t)((i / S) & 1), prm.err, prm.wait_ns)) { ok = false; break; }
      const uint32_t wt = smem_u32(smem + (size_t)st * C::kStage);
      const uint32_t tt = wt + C::kWTile;     // the token tile
      const uint32_t at = C::kWA ? wt : tt;    // the A and B operands' tiles
      const uint32_t bt = C::kWA ? tt : wt;
      float p[4][C::kMF][4];                   // Block_FP8: this group's partial sums
      if constexpr (FMT == kBLOCK) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int mf = 0; mf < C::kMF; ++mf)
#pragma unroll
            for (int j = 0; j < 4; ++j) p[q][mf][j] = 0.f;
      }
#pragma unroll
      for (int kp = 0; kp < 2; ++kp) {        // pairs of 32-byte K steps
        uint32_t b[4];
        {
          const int c = 4 * kp + bchk;
          ldsm_x4(bt + (uint32_t)(brow * kKTileBytes + ((c ^ (brow & 7)) << 4)), b[0], b[1], b[2], b[3]);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {         // K step 2 kp + h
#pragma unroll
          for (int mf = 0; mf < C::kMF; ++mf) {
            const int r = mf * 16 + arow;
            const int c = 2 * (2 * kp + h) + achk;
            uint32_t a[4];
            ldsm_x4(at + (uint32_t)(r * kKTileBytes + ((c ^ (r & 7)) << 4)), a[0], a[1], a[2], a[3]);
            if constexpr (kInt) {
              mma16832_s8(reinterpret_cast<int(&)[4]>(acc[2 * kp + h][mf]), a, b[2 * h], b[2 * h + 1]);
            } else if constexpr (FMT == kBLOCK) {
              mma16832_e4m3(p[2 * kp + h][mf], a, b[2 * h], b[2 * h + 1]);
            } else {
              mma16832_e4m3(reinterpret_cast<float(&)[4]>(acc[2 * kp + h][mf]), a, b[2 * h], b[2 * h + 1]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);  // slot free for the producer
      if constexpr (FMT == kBLOCK) {
        // promotion of this 128-K group: acc += p_g * (s_a[token, g] * s_w[block, g]),
        // p_g the group's sum of its four K steps; the promoted sums of a
        // warp's groups alternate over two accumulator sets
        const int q = (i / C::kKG) & 1;
#pragma unroll
        for (int mf = 0; mf < C::kMF; ++mf) {
          const float flo = sa_lo[mf] * sw, fhi = sa_hi[mf] * sw;
          float* af = reinterpret_cast<float*>(acc[q][mf]);
          float pg[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) pg[j] = (p[0][mf][j] + p[1][mf][j]) + (p[2][mf][j] + p[3][mf][j]);
          // element j: row g (j < 2) or g + 8, column 2t + (j & 1); the token
          // is the row (tokens as A) or the column (weights as A)
          const float f0 = flo, f1 = C::kWA ? fhi : flo, f2 = C::kWA ? flo : fhi, f3 = fhi;
          af[0] = fmaf(pg[0], f0, af[0]);
          af[1] = fmaf(pg[1], f1, af[1]);
          af[2] = fmaf(pg[2], f2, af[2]);
          af[3] = fmaf(pg[3], f3, af[3]);
        }
      }
    }
    // ---- this warp's sum in a fixed order, then the K groups meet in
    // shared memory
#pragma unroll
    for (int mf = 0; mf < C::kMF; ++mf) {
      Acc v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = (acc[0][mf][j] + acc[1][mf][j]) + (acc[2][mf][j] + acc[3][mf][j]);
      Acc* rw = red + ((size_t)(warp * C::kMF + mf) * 16) * 8;
      rw[g * 8 + 2 * t] = v[0];
      rw[g * 8 + 2 * t + 1] = v[1];
      rw[(g + 8) * 8 + 2 * t] = v[2];
      rw[(g + 8) * 8 + 2 * t + 1] = v[3];
    }
  }
  // every thread (the producer warp too) meets here; a thread that gave up on
  // a wait leaves no sum, and then the epilogue stores nothing
  const int all_ok = __syncthreads_and(ok ? 1 : 0);
  if (warp < C::kWarps) {
    if (all_ok) {
      // ---- epilogue: one unit = 8 consecutive channels of one token
      const int etid = threadIdx.x;            // 0 .. 255
      const bool vec = (prm.ldy % 8) == 0;
      for (int u = etid; u < TM * NF; u += 32 * C::kWarps) {
        const int mm = u / NF, nfu = u % NF;
        const int m = m0 + mm, nb = n0 + nfu * 8;
        if (m >= prm.M || nb >= prm.N) continue;
        Acc s8[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) s8[j] = (Acc)0;
        for (int k2 = 0; k2 < C::kKG; ++k2) {  // K-group order: deterministic
          if constexpr (C::kWA) {
            // warp (k2, nfu / 2), fragment rows 8 (nfu % 2) + j, column mm
            const Acc* rw = red + (size_t)(k2 * C::kUnits + nfu / 2) * 128 + (nfu % 2) * 64 + mm;
#pragma unroll
            for (int j = 0; j < 8; ++j) s8[j] += rw[j * 8];
          } else {
            const int mf = mm / 16, rr = mm % 16;
            const Acc* rw = red + ((size_t)((k2 * NF + nfu) * C::kMF + mf) * 16 + rr) * 8;
#pragma unroll
            for (int j = 0; j < 8; ++j) s8[j] += rw[j];
          }
        }
        if (prm.out_kind == 1) {
          uint32_t* Yu = reinterpret_cast<uint32_t*>(prm.Y) + (size_t)m * prm.ldy;
          for (int j = 0; j < 8 && nb + j < prm.N; ++j) Yu[nb + j] = *reinterpret_cast<const uint32_t*>(&s8[j]);
          continue;
        }
        float y8[8];
        if constexpr (FMT == kBLOCK) {
#pragma unroll
          for (int j = 0; j < 8; ++j) y8[j] = s8[j];
        } else {
          const float sa = __ldg(prm.scale_a + m);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float sw = (nb + j < prm.N) ? __ldg(prm.scale_w + nb + j) : 0.f;
            y8[j] = kInt ? (__int2float_rn((int)s8[j]) * sa) * sw : ((float)s8[j] * sa) * sw;
          }
        }
        __nv_bfloat16* Yb = reinterpret_cast<__nv_bfloat16*>(prm.Y) + (size_t)m * prm.ldy;
        if (vec && nb + 8 <= prm.N) {
          uint32_t pk[4];
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(y8[2 * h], y8[2 * h + 1]);
            pk[h] = *reinterpret_cast<const uint32_t*>(&b2);
          }
          *reinterpret_cast<uint4*>(Yb + nb) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        } else {
          for (int j = 0; j < 8 && nb + j < prm.N; ++j) Yb[nb + j] = __float2bfloat16_rn(y8[j]);
        }
      }
    }
    if (threadIdx.x == 0) trace_at(prm, kTrDone);
  }
}

}  // namespace qg
