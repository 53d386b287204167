// gemm_nvf4.cu — instantiations of the unified GEMM kernel for one format.
#define QG_FMT qg::kNVF4
#define QG_LAUNCH_NAME launch_gemm_nvf4
#include "gemm_launch.cuh"
