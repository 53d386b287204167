// gemm_block.cu — instantiations of the unified GEMM kernel for one format.
#define QG_FMT qg::kBLOCK
#define QG_LAUNCH_NAME launch_gemm_block
#include "gemm_launch.cuh"
