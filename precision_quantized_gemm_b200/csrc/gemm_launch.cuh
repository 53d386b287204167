// gemm_launch.cuh — host-side launch of one format's GEMM instantiations.
// Included by exactly one translation unit per format with QG_FMT and
// QG_LAUNCH_NAME defined.  A format whose grouped (mixture-of-experts)
// kernels live in a unit of their own defines QG_GROUPED_OWN_UNIT in the
// format's unit and QG_GROUPED_ONLY in that second unit (the two compile in
// parallel).
#pragma once
#include <atomic>
#include "attr_cache.h"
#include "gemm_kernel.cuh"
#include "internal.h"
#include "pair.cuh"
#include "persist.cuh"
#include "skinny.cuh"

#define QG_CAT2(a, b) a##b
#define QG_CAT(a, b) QG_CAT2(a, b)

namespace qg {
namespace {

template <int FMT, bool SWAP, int BN, bool FUSED, bool GROUPED>
cudaError_t launch_one(const CUtensorMap& tp, const CUtensorMap& tq, const CUtensorMap& ty,
                       const GemmParams& prm,
                       dim3 grid, cudaStream_t st, bool pdl) {
  auto kern = qgemm_kernel<FMT, SWAP, BN, FUSED, GROUPED>;
  const int act_tiles = FUSED ? prm.nkt_max : 0;
  size_t smem = smem_bytes<FMT, SWAP, BN>(prm.stages, prm.nkt_max, prm.recv_cols, act_tiles);
  // Every CTA of this kernel that fits on an SM must also fit in its 512 TMEM
  // columns: a CTA whose tcgen05.alloc waited on another CTA of the same
  // (clustered) grid could wait for good.  At most 512 / kTmemCols CTAs may
  // share an SM, so the shared memory of one is raised to at least
  // 228 KB / (that count + 1).
  constexpr int kTmemCtas = 512 / tmem_cols<FMT, SWAP, BN, FUSED, GROUPED>();
  const size_t smem_floor = (size_t)233472 / (kTmemCtas + 1);
  if (smem < smem_floor) smem = smem_floor;
  // the kernel's shared-memory limit is raised per device (the attribute
  // acts on the current device), once per larger size
  static GrowOnlyAttr smem_attr;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = static_cast<cudaError_t>(smem_attr.ensure(dev, (int)smem, [&](int bytes) {
    return static_cast<int>(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  }));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(Cfg<FMT, BN>::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (prm.split_k > 1 && prm.reduce_mode == kReduceCluster) {
    // the split_k CTAs of one output tile form one cluster along z
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 1;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = prm.split_k;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, tp, tq, ty, prm);
}

template <int FMT, bool SWAP, bool FUSED, bool GROUPED = false>
cudaError_t launch_bn(int bn, const CUtensorMap& tp, const CUtensorMap& tq, const CUtensorMap& ty,
                      const GemmParams& prm,
                      dim3 grid, cudaStream_t st, bool pdl) {
  switch (bn) {
    case 16: return launch_one<FMT, SWAP, 16, FUSED, GROUPED>(tp, tq, ty, prm, grid, st, pdl);
    case 32: return launch_one<FMT, SWAP, 32, FUSED, GROUPED>(tp, tq, ty, prm, grid, st, pdl);
    case 64: return launch_one<FMT, SWAP, 64, FUSED, GROUPED>(tp, tq, ty, prm, grid, st, pdl);
    case 128: return launch_one<FMT, SWAP, 128, FUSED, GROUPED>(tp, tq, ty, prm, grid, st, pdl);
    case 256: return launch_one<FMT, SWAP, 256, FUSED, GROUPED>(tp, tq, ty, prm, grid, st, pdl);
    default: return cudaErrorInvalidValue;
  }
}

// Bytes from the ring's start to the end of the Q tiles: the region the
// epilogue reuses once the mainloop is done (act_tiles > 0: the Q tiles are
// the thread-written activation slice instead of one per stage).
template <int FMT, int BN>
size_t ring_bytes(int stages, int act_tiles) {
  using C = Cfg<FMT, BN>;
  return (size_t)stages * kPTileBytes + (size_t)(act_tiles > 0 ? act_tiles : stages) * C::kQTileBytes;
}

template <int FMT, int BN>
bool cluster_fits(bool swap, int stages, int act_tiles) {
  return (size_t)(swap ? red_bytes<true, BN>() : red_bytes<false, BN>()) <= ring_bytes<FMT, BN>(stages, act_tiles);
}

template <int FMT>
bool cluster_fits_for(int bn, bool swap, int stages, int act_tiles) {
  switch (bn) {
    case 16: return cluster_fits<FMT, 16>(swap, stages, act_tiles);
    case 32: return cluster_fits<FMT, 32>(swap, stages, act_tiles);
    case 64: return cluster_fits<FMT, 64>(swap, stages, act_tiles);
    case 128: return cluster_fits<FMT, 128>(swap, stages, act_tiles);
    case 256: return cluster_fits<FMT, 256>(swap, stages, act_tiles);
    default: return false;
  }
}

// Shared memory of a launch; configurations whose output tile does not fit
// the ring region (reused by the epilogue) report an impossible size.
template <int FMT, bool SWAP, int BN>
size_t smem_checked(int stages, int nkt_max, int recv_cols, int act_tiles) {
  if ((size_t)tile_bytes<SWAP, BN>() > ring_bytes<FMT, BN>(stages, act_tiles)) return (size_t)1 << 30;
  return smem_bytes<FMT, SWAP, BN>(stages, nkt_max, recv_cols, act_tiles);
}

template <int FMT, bool SWAP>
size_t smem_for(int bn, int stages, int nkt_max, int recv_cols, int act_tiles) {
  switch (bn) {
    case 16: return smem_checked<FMT, SWAP, 16>(stages, nkt_max, recv_cols, act_tiles);
    case 32: return smem_checked<FMT, SWAP, 32>(stages, nkt_max, recv_cols, act_tiles);
    case 64: return smem_checked<FMT, SWAP, 64>(stages, nkt_max, recv_cols, act_tiles);
    case 128: return smem_checked<FMT, SWAP, 128>(stages, nkt_max, recv_cols, act_tiles);
    case 256: return smem_checked<FMT, SWAP, 256>(stages, nkt_max, recv_cols, act_tiles);
    default: return (size_t)1 << 30;
  }
}

template <int FMT, int TM, int NF>
cudaError_t launch_skinny_one(const CUtensorMap& tw, const CUtensorMap& ta, const GemmParams& prm, dim3 grid,
                              cudaStream_t st, bool pdl) {
  auto kern = qgemm_skinny_kernel<FMT, TM, NF>;
  const size_t smem = skinny_smem_bytes<FMT, TM, NF>(prm.stages);
  static GrowOnlyAttr smem_attr;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = static_cast<cudaError_t>(smem_attr.ensure(dev, (int)smem, [&](int bytes) {
    return static_cast<int>(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  }));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(SkCfg<FMT, TM, NF>::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, tw, ta, prm);
}

template <int FMT, int TM>
cudaError_t launch_skinny_rows(int rows, const CUtensorMap& tw, const CUtensorMap& ta, const GemmParams& prm,
                               dim3 grid, cudaStream_t st, bool pdl) {
  switch (rows) {
    case 8:
      if constexpr (TM == 8) return cudaErrorInvalidValue;
      else return launch_skinny_one<FMT, TM, 1>(tw, ta, prm, grid, st, pdl);
    case 16: return launch_skinny_one<FMT, TM, 2>(tw, ta, prm, grid, st, pdl);
    case 32: return launch_skinny_one<FMT, TM, 4>(tw, ta, prm, grid, st, pdl);
    case 64: return launch_skinny_one<FMT, TM, 8>(tw, ta, prm, grid, st, pdl);
    default: return cudaErrorInvalidValue;
  }
}

template <int FMT, int BN>
cudaError_t launch_persist_one(const CUtensorMap& tp, const CUtensorMap& tq, const CUtensorMap& ty,
                               const GemmParams& prm, dim3 grid, cudaStream_t st, bool pdl) {
  auto kern = qgemm_persist_kernel<FMT, BN>;
  size_t smem = ps_smem_bytes<FMT, BN>(prm.stages);
  // at most 512 / (2 BN) CTAs fit an SM's TMEM: the shared memory keeps it so
  constexpr int kTmemCtas = 512 / PsCfg<FMT, BN>::kTmemCols;
  const size_t smem_floor = (size_t)233472 / (kTmemCtas + 1);
  if (smem < smem_floor) smem = smem_floor;
  static GrowOnlyAttr smem_attr;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = static_cast<cudaError_t>(smem_attr.ensure(dev, (int)smem, [&](int bytes) {
    return static_cast<int>(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  }));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(PsCfg<FMT, BN>::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, tp, tq, ty, prm);
}

template <int BN>
cudaError_t launch_persist_block_one(const CUtensorMap& tp, const CUtensorMap& tq, const CUtensorMap& ty,
                                     const GemmParams& prm, dim3 grid, cudaStream_t st, bool pdl) {
  auto kern = qgemm_persist_block_kernel<BN>;
  if constexpr (PbCfg<BN>::kRegSplit) {
    // setmaxnreg.inc waits until the new counts fit the CTA's launch
    // allocation: launch only the build whose count the split was sized for
    static std::atomic<int> regs{0};
    int r = regs.load(std::memory_order_relaxed);
    if (r == 0) {
      cudaFuncAttributes fa;
      const cudaError_t e0 = cudaFuncGetAttributes(&fa, kern);
      if (e0 != cudaSuccess) return e0;
      r = fa.numRegs;
      regs.store(r, std::memory_order_relaxed);
    }
    if (r != PbCfg<BN>::kRegsLaunch) return cudaErrorInvalidValue;
  }
  size_t smem = pb_smem_bytes<BN>(prm.stages, prm.kt_total);
  // the group buffers take all 512 TMEM columns: one CTA per SM
  const size_t smem_floor = (size_t)233472 / 2;
  if (smem < smem_floor) smem = smem_floor;
  static GrowOnlyAttr smem_attr;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = static_cast<cudaError_t>(smem_attr.ensure(dev, (int)smem, [&](int bytes) {
    return static_cast<int>(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  }));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(PbCfg<BN>::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, tp, tq, ty, prm);
}

// Block_FP8 on CTA pairs (variant 3): clusters of two along x, one CTA per
// SM (the pair's TMEM takes all 512 columns of each).
template <int BN>
cudaError_t launch_pair_block(const CUtensorMap& tp, const CUtensorMap& tq, const CUtensorMap& ty,
                              const GemmParams& prm, dim3 grid, cudaStream_t st, bool pdl) {
  auto kern = qgemm_pair_block_kernel<BN>;
  {
    // setmaxnreg.inc waits until the new counts fit the CTA's launch
    // allocation: launch only the build whose count the split was sized for
    static std::atomic<int> regs{0};
    int r = regs.load(std::memory_order_relaxed);
    if (r == 0) {
      cudaFuncAttributes fa;
      const cudaError_t e0 = cudaFuncGetAttributes(&fa, kern);
      if (e0 != cudaSuccess) return e0;
      r = fa.numRegs;
      regs.store(r, std::memory_order_relaxed);
    }
    if (r != PpCfg<BN>::kRegsLaunch) return cudaErrorInvalidValue;
  }
  size_t smem = pp_smem_bytes<BN>(prm.stages);
  const size_t smem_floor = (size_t)233472 / 2;
  if (smem < smem_floor) smem = smem_floor;
  static GrowOnlyAttr smem_attr;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = static_cast<cudaError_t>(smem_attr.ensure(dev, (int)smem, [&](int bytes) {
    return static_cast<int>(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  }));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(PpCfg<BN>::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, tp, tq, ty, prm);
}

template <int FMT, int TM>
size_t skinny_smem_rows(int rows, int stages) {
  switch (rows) {
    case 8:
      if constexpr (TM == 8) return (size_t)1 << 30;
      else return skinny_smem_bytes<FMT, TM, 1>(stages);
    case 16: return skinny_smem_bytes<FMT, TM, 2>(stages);
    case 32: return skinny_smem_bytes<FMT, TM, 4>(stages);
    case 64: return skinny_smem_bytes<FMT, TM, 8>(stages);
    default: return (size_t)1 << 30;
  }
}

}  // namespace

#if !defined(QG_GROUPED_OWN_UNIT) || defined(QG_GROUPED_ONLY)
// grouped (mixture-of-experts) launch: Swap-AB, activations by TMA
cudaError_t QG_CAT(QG_LAUNCH_NAME, _grouped)(int tile_n, const CUtensorMap& tp, const CUtensorMap& tq,
                                             const CUtensorMap& ty,
                                             const GemmParams& prm, dim3 grid, cudaStream_t st, bool pdl) {
  return launch_bn<QG_FMT, true, false, true>(tile_n, tp, tq, ty, prm, grid, st, pdl);
}
#endif

#ifndef QG_GROUPED_ONLY
cudaError_t QG_CAT(QG_LAUNCH_NAME, _skinny)(int tile_n, int rows, const CUtensorMap& tw, const CUtensorMap& ta,
                                            const GemmParams& prm, dim3 grid, cudaStream_t st, bool pdl) {
  if constexpr (QG_FMT == kNVF4) {
    return cudaErrorInvalidValue;
  } else {
    if (tile_n == 8) return launch_skinny_rows<QG_FMT, 8>(rows, tw, ta, prm, grid, st, pdl);
    if (tile_n == 16) return launch_skinny_rows<QG_FMT, 16>(rows, tw, ta, prm, grid, st, pdl);
    if (tile_n == 32) return launch_skinny_rows<QG_FMT, 32>(rows, tw, ta, prm, grid, st, pdl);
    return cudaErrorInvalidValue;
  }
}

// The persistent kernel (variant 2): FP8_Dynamic, W8A8_INT8 and Block_FP8,
// tile_n 128 or 256.
cudaError_t QG_CAT(QG_LAUNCH_NAME, _persist)(int tile_n, const CUtensorMap& tp, const CUtensorMap& tq,
                                             const CUtensorMap& ty, const GemmParams& prm, dim3 grid,
                                             cudaStream_t st, bool pdl) {
  if constexpr (QG_FMT == kFP8 || QG_FMT == kINT8) {
    if (tile_n == 128) return launch_persist_one<QG_FMT, 128>(tp, tq, ty, prm, grid, st, pdl);
    if (tile_n == 256) return launch_persist_one<QG_FMT, 256>(tp, tq, ty, prm, grid, st, pdl);
  } else if constexpr (QG_FMT == kBLOCK) {
    if (tile_n == 128) return launch_persist_block_one<128>(tp, tq, ty, prm, grid, st, pdl);
    if (tile_n == 256) return launch_persist_block_one<256>(tp, tq, ty, prm, grid, st, pdl);
  }
  return cudaErrorInvalidValue;
}

// Block_FP8 on CTA pairs (variant 3): pair tiles of 256 x 128 or 256 x 256.
cudaError_t QG_CAT(QG_LAUNCH_NAME, _pair)(int tile_n, const CUtensorMap& tp, const CUtensorMap& tq,
                                          const CUtensorMap& ty, const GemmParams& prm, dim3 grid,
                                          cudaStream_t st, bool pdl) {
  if constexpr (QG_FMT == kBLOCK) {
    if (tile_n == 128) return launch_pair_block<128>(tp, tq, ty, prm, grid, st, pdl);
    if (tile_n == 256) return launch_pair_block<256>(tp, tq, ty, prm, grid, st, pdl);
  }
  return cudaErrorInvalidValue;
}

size_t QG_CAT(QG_LAUNCH_NAME, _pair_smem)(int tile_n, int stages, int nkt) {
  (void)nkt;
  if constexpr (QG_FMT == kBLOCK) {
    if (tile_n == 128) return pp_smem_bytes<128>(stages);
    if (tile_n == 256) return pp_smem_bytes<256>(stages);
  }
  return (size_t)1 << 30;
}

size_t QG_CAT(QG_LAUNCH_NAME, _persist_smem)(int tile_n, int stages, int nkt) {
  if constexpr (QG_FMT == kFP8 || QG_FMT == kINT8) {
    if (tile_n == 128) return ps_smem_bytes<QG_FMT, 128>(stages);
    if (tile_n == 256) return ps_smem_bytes<QG_FMT, 256>(stages);
  } else if constexpr (QG_FMT == kBLOCK) {
    if (tile_n == 128) return pb_smem_bytes<128>(stages, nkt);
    if (tile_n == 256) return pb_smem_bytes<256>(stages, nkt);
  }
  return (size_t)1 << 30;
}

size_t QG_CAT(QG_LAUNCH_NAME, _skinny_smem)(int tile_n, int rows, int stages) {
  if constexpr (QG_FMT == kNVF4) {
    return (size_t)1 << 30;
  } else {
    if (tile_n == 8) return skinny_smem_rows<QG_FMT, 8>(rows, stages);
    if (tile_n == 16) return skinny_smem_rows<QG_FMT, 16>(rows, stages);
    if (tile_n == 32) return skinny_smem_rows<QG_FMT, 32>(rows, stages);
    return (size_t)1 << 30;
  }
}

cudaError_t QG_LAUNCH_NAME(bool swap, int tile_n, const CUtensorMap& tp, const CUtensorMap& tq,
                           const CUtensorMap& ty,
                           const GemmParams& prm, dim3 grid, cudaStream_t st, bool pdl) {
  if (prm.expert_offsets != nullptr) {
    if (swap && prm.a_mode == kActTma) return QG_CAT(QG_LAUNCH_NAME, _grouped)(tile_n, tp, tq, ty, prm, grid, st, pdl);
    return cudaErrorInvalidValue;
  }
  if (prm.a_mode == kActFused) {
    // fused activation quantisation: Swap-AB, 8-bit formats only
    if constexpr (QG_FMT != kNVF4) {
      if (swap) return launch_bn<QG_FMT, true, true>(tile_n, tp, tq, ty, prm, grid, st, pdl);
    }
    return cudaErrorInvalidValue;
  }
  return swap ? launch_bn<QG_FMT, true, false>(tile_n, tp, tq, ty, prm, grid, st, pdl)
              : launch_bn<QG_FMT, false, false>(tile_n, tp, tq, ty, prm, grid, st, pdl);
}

size_t QG_CAT(QG_LAUNCH_NAME, _smem)(int tile_n, bool swap, int stages, int nkt_max, int recv_cols,
                                     int act_tiles) {
  return swap ? smem_for<QG_FMT, true>(tile_n, stages, nkt_max, recv_cols, act_tiles)
              : smem_for<QG_FMT, false>(tile_n, stages, nkt_max, recv_cols, act_tiles);
}

bool QG_CAT(QG_LAUNCH_NAME, _cluster_fits)(int tile_n, bool swap, int stages, int act_tiles) {
  return cluster_fits_for<QG_FMT>(tile_n, swap, stages, act_tiles);
}

cudaError_t QG_CAT(QG_LAUNCH_NAME, _reduce)(const GemmParams& prm, cudaStream_t st, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  const long long mn = (long long)prm.M * prm.N;
  long long blocks = (mn + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  cfg.gridDim = dim3((unsigned)(blocks < 1 ? 1 : blocks));
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, splitk_reduce_kernel<QG_FMT>, prm);
}

#endif  // QG_GROUPED_ONLY

}  // namespace qg
