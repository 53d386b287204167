// gemm_nvf4_grouped.cu — the grouped (mixture-of-experts) NVFP4 kernels.
#define QG_FMT qg::kNVF4
#define QG_LAUNCH_NAME launch_gemm_nvf4
#define QG_GROUPED_OWN_UNIT
#define QG_GROUPED_ONLY
#include "gemm_launch.cuh"
