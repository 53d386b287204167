// gemm_fp8.cu — instantiations of the unified GEMM kernel for one format.
#define QG_FMT qg::kFP8
#define QG_LAUNCH_NAME launch_gemm_fp8
#include "gemm_launch.cuh"
