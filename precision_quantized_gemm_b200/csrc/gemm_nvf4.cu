// gemm_nvf4.cu — instantiations of the unified GEMM kernel for one format
// (its grouped kernels: gemm_nvf4_grouped.cu).
#define QG_FMT qg::kNVF4
#define QG_LAUNCH_NAME launch_gemm_nvf4
#define QG_GROUPED_OWN_UNIT
#include "gemm_launch.cuh"
