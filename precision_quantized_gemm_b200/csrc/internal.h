// internal.h — declarations shared by the library's translation units.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace qg {

struct GemmParams;

}  // namespace qg
#include "../../include/qgemm.h"
namespace qg {

qg_status check_run_args(qg_format f, const qg_operand* A, const qg_operand* W, int M, int N, int K,
                         const qg_config* cfg, void* workspace, size_t ws_bytes, void* Y, int ldy,
                         int out_kind);

constexpr int kNvfp4AmaxMaxCtas = 296;   // partial-amax slots in the NVFP4 quant workspace

// Configuration feasibility (the checks of qgemm_run), the shared memory a
// launch takes, the SM count of the current device (148 without one), the
// fixed-rule default configuration (api.cu).
qg_status config_check(qg_format f, int M, int N, int K, const qg_config* c);
size_t config_smem(qg_format f, int M, int K, const qg_config* c);
int device_sm_count();
qg_status rule_default_config(qg_format f, int M, int N, int K, qg_config* out);
// The candidate grid the scorer ranks and the tuner times (scorer.cu), before
// feasibility checks.
void candidate_grid(qg_format f, int M, int N, int K, qg_config* out, int max_out, int* n_out);

cudaError_t launch_quant_rows(bool int8, const void* X, int R, int K, int ldx, void* q,
                              float* scale, cudaStream_t st, bool pdl);
cudaError_t launch_quant_act_groups(const void* X, int M, int K, int ldx, void* q, float* scale,
                                    cudaStream_t st, bool pdl);
cudaError_t launch_quant_weight_blocks(const void* W, int N, int K, void* q, float* scale,
                                       cudaStream_t st, bool pdl);
int nvfp4_amax_ctas(int R, int K);
cudaError_t launch_quant_nvfp4(const void* X, int R, int K, int ldx, const float* static_amax,
                               void* q, void* sf, float* gscale, float* partial,
                               cudaStream_t st, bool pdl, const int* offsets = nullptr,
                               int experts = 0);

// GEMM launchers, one per format (each in its own translation unit).
// Returns cudaErrorInvalidValue for a (swap, tile_n) pair not instantiated.
#define QG_DECLARE_GEMM_LAUNCH(NAME)                                                      \
  cudaError_t NAME(bool swap, int tile_n, const CUtensorMap& tp, const CUtensorMap& tq,    \
                   const CUtensorMap& ty,                                                  \
                   const GemmParams& prm, dim3 grid, cudaStream_t st, bool pdl);           \
  size_t NAME##_smem(int tile_n, bool swap, int stages, int nkt_max, int recv_cols,        \
                     int act_tiles);                                                       \
  bool NAME##_cluster_fits(int tile_n, bool swap, int stages, int act_tiles);              \
  cudaError_t NAME##_reduce(const GemmParams& prm, cudaStream_t st, bool pdl);             \
  cudaError_t NAME##_grouped(int tile_n, const CUtensorMap& tp, const CUtensorMap& tq,     \
                             const CUtensorMap& ty,                                        \
                             const GemmParams& prm, dim3 grid, cudaStream_t st, bool pdl); \
  cudaError_t NAME##_skinny(int tile_n, int rows, const CUtensorMap& tw, const CUtensorMap& ta, \
                            const GemmParams& prm, dim3 grid, cudaStream_t st, bool pdl);     \
  size_t NAME##_skinny_smem(int tile_n, int rows, int stages);                              \
  cudaError_t NAME##_persist(int tile_n, const CUtensorMap& tp, const CUtensorMap& tq,     \
                             const CUtensorMap& ty, const GemmParams& prm, dim3 grid,      \
                             cudaStream_t st, bool pdl);                                   \
  size_t NAME##_persist_smem(int tile_n, int stages, int nkt);                              \
  cudaError_t NAME##_pair(int tile_n, const CUtensorMap& tp, const CUtensorMap& tq,        \
                          const CUtensorMap& ty, const GemmParams& prm, dim3 grid,         \
                          cudaStream_t st, bool pdl);                                      \
  size_t NAME##_pair_smem(int tile_n, int stages, int nkt);
QG_DECLARE_GEMM_LAUNCH(launch_gemm_fp8)
QG_DECLARE_GEMM_LAUNCH(launch_gemm_int8)
QG_DECLARE_GEMM_LAUNCH(launch_gemm_block)
QG_DECLARE_GEMM_LAUNCH(launch_gemm_nvf4)
#undef QG_DECLARE_GEMM_LAUNCH

}  // namespace qg
