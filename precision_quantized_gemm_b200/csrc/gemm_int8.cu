// gemm_int8.cu — instantiations of the unified GEMM kernel for one format.
#define QG_FMT qg::kINT8
#define QG_LAUNCH_NAME launch_gemm_int8
#include "gemm_launch.cuh"
