// api.cu — the C ABI of libqgemm.so: argument checks, buffer sizes, TMA
// descriptors, launches of the quantisers and of the unified GEMM kernel.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/qgemm.h"
#include "gemm_kernel.cuh"
#include "internal.h"

namespace qg {
// Device error word: set by bounded in-kernel waits that expire.
__device__ unsigned int g_qg_error = 0;
}  // namespace qg

namespace {

using qg::GemmParams;

bool g_pdl = true;
unsigned long long g_wait_ns = qg::kWaitLimitNs;   // limit of every in-kernel wait
bool g_l2_ahead = true;                           // Swap-AB weight prefetch for later CTAs
bool g_tma_store = true;                          // TMA stores of direct standard-orientation tiles
unsigned long long* g_trace = nullptr;   // debug phase trace buffer (device)
size_t g_trace_bytes = 0;

constexpr int kMaxDevices = 64;
struct DeviceInfo {
  bool probed = false;
  bool sm100 = false;
  int sms = 0;
  unsigned int* err = nullptr;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

qg_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QG_ERR_NO_DEVICE;
  if (dev < 0 || dev >= kMaxDevices) return QG_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.probed) {
    cudaDeviceProp p;
    if (cudaGetDeviceProperties(&p, dev) != cudaSuccess) return QG_ERR_CUDA;
    d.sm100 = (p.major == 10 && p.minor == 0);
    d.sms = p.multiProcessorCount;
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, qg::g_qg_error) != cudaSuccess) return QG_ERR_CUDA;
    d.err = static_cast<unsigned int*>(addr);
    d.probed = true;
  }
  if (!d.sm100) return QG_ERR_UNSUPPORTED;
  *out = &d;
  return QG_OK;
}

// One mbarrier that nothing arrives on, waited for with the library's own
// bounded wait: after `limit_ns` the wait gives up and sets the device error
// word, exactly as a GEMM's wait would.  No copy or MMA is in flight, so the
// kernel then simply returns.
__global__ void wait_expiry_kernel(unsigned int* err, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    qg::mbar_init(&bar, 1);
    qg::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)qg::mbar_wait(&bar, 0, err, limit_ns);
  __syncthreads();
}

// ------------------------------------------------------------- TMA maps --
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2D byte tensor [rows, row_bytes] (row stride row_bytes), box 128 bytes x
// box_rows, 128-byte swizzle, out-of-range elements read as zero.
bool make_tmap(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows,
               uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {row_bytes, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The bf16 output y [M, ldy] as a 2D byte tensor of N * 2 bytes per row, read
// in boxes of 128 rows x 128 bytes (64 channels) with the 128-byte swizzle:
// the tile-store map of the direct epilogue.
bool make_tmap_y(CUtensorMap* m, const void* Y, int N, int M, int ldy) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)N * 2, (cuuint64_t)M};
  cuuint64_t strides[1] = {(cuuint64_t)ldy * 2};
  cuuint32_t box[2] = {128, 128};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(Y), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- checks --
bool valid_format(int f) { return f >= QG_FP8_DYNAMIC && f <= QG_NVFP4; }
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
int k_multiple(qg_format f) {
  switch (f) {
    case QG_BLOCK_FP8: return 128;
    case QG_NVFP4: return 32;
    default: return 16;
  }
}
size_t row_bytes(qg_format f, int K) { return f == QG_NVFP4 ? (size_t)K / 2 : (size_t)K; }
int kt_total(qg_format f, int K) { return (int)((row_bytes(f, K) + 127) / 128); }
bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// How the activation tiles of a launch fill (qg::kAct*): fused launches
// quantise the bf16 activations in the kernel; every other launch streams the
// quantised codes through the ring by TMA.
int act_mode(bool fused) { return fused ? qg::kActFused : qg::kActTma; }

// Launch-dependent parts of the shared-memory carve-up: the K tiles of the
// longest split slice (Block_FP8 stages that many scale columns; a fused
// launch's activation slice that many tiles) and the token columns of a
// push-mode cluster receive slot (only real tokens are pushed).
struct LaunchShape {
  int nkt_max;
  int recv_cols;
  int a_mode;
  int act_tiles;
};
LaunchShape launch_shape(qg_format f, int M, int K, const qg_config* c, bool fused) {
  LaunchShape ls;
  const int kt = kt_total(f, K);
  ls.nkt_max = (kt + c->split_k - 1) / c->split_k;
  const bool push = c->split_k > 1 && c->reduce_mode == qg::kReduceCluster && c->tile_n <= 64;
  ls.recv_cols = push ? (c->swap_ab ? (M < c->tile_n ? M : c->tile_n) : c->tile_n) : 0;
  ls.a_mode = act_mode(fused);
  ls.act_tiles = ls.a_mode != qg::kActTma ? ls.nkt_max : 0;
  return ls;
}

size_t skinny_smem(qg_format f, const qg_config* c) {
  switch (f) {
    case QG_FP8_DYNAMIC: return qg::launch_gemm_fp8_skinny_smem(c->tile_n, c->rows, c->stages);
    case QG_W8A8_INT8: return qg::launch_gemm_int8_skinny_smem(c->tile_n, c->rows, c->stages);
    case QG_BLOCK_FP8: return qg::launch_gemm_block_skinny_smem(c->tile_n, c->rows, c->stages);
    default: return (size_t)1 << 30;
  }
}

size_t persist_smem(qg_format f, int K, const qg_config* c) {
  const int nkt = kt_total(f, K);
  switch (f) {
    case QG_FP8_DYNAMIC: return qg::launch_gemm_fp8_persist_smem(c->tile_n, c->stages, nkt);
    case QG_W8A8_INT8: return qg::launch_gemm_int8_persist_smem(c->tile_n, c->stages, nkt);
    case QG_BLOCK_FP8: return qg::launch_gemm_block_persist_smem(c->tile_n, c->stages, nkt);
    default: return (size_t)1 << 30;
  }
}

size_t pair_smem(qg_format f, int K, const qg_config* c) {
  if (f != QG_BLOCK_FP8) return (size_t)1 << 30;
  return qg::launch_gemm_block_pair_smem(c->tile_n, c->stages, kt_total(f, K));
}

size_t gemm_smem(qg_format f, int M, int K, const qg_config* c, bool fused) {
  if (c->variant == 1) return skinny_smem(f, c);
  if (c->variant == 2) return persist_smem(f, K, c);
  if (c->variant == 3) return pair_smem(f, K, c);
  const LaunchShape ls = launch_shape(f, M, K, c, fused);
  const bool swap = c->swap_ab != 0;
  const int tn = c->tile_n, st = c->stages;
  switch (f) {
    case QG_FP8_DYNAMIC: return qg::launch_gemm_fp8_smem(tn, swap, st, ls.nkt_max, ls.recv_cols, ls.act_tiles);
    case QG_W8A8_INT8: return qg::launch_gemm_int8_smem(tn, swap, st, ls.nkt_max, ls.recv_cols, ls.act_tiles);
    case QG_BLOCK_FP8: return qg::launch_gemm_block_smem(tn, swap, st, ls.nkt_max, ls.recv_cols, ls.act_tiles);
    default: return qg::launch_gemm_nvf4_smem(tn, swap, st, ls.nkt_max, ls.recv_cols, ls.act_tiles);
  }
}
constexpr size_t kSmemLimit = 232448;  // 227 KB opt-in per CTA on sm_100

bool cluster_fits(qg_format f, int M, int K, const qg_config* c, bool fused) {
  const int act_tiles = launch_shape(f, M, K, c, fused).act_tiles;
  const bool swap = c->swap_ab != 0;
  switch (f) {
    case QG_FP8_DYNAMIC: return qg::launch_gemm_fp8_cluster_fits(c->tile_n, swap, c->stages, act_tiles);
    case QG_W8A8_INT8: return qg::launch_gemm_int8_cluster_fits(c->tile_n, swap, c->stages, act_tiles);
    case QG_BLOCK_FP8: return qg::launch_gemm_block_cluster_fits(c->tile_n, swap, c->stages, act_tiles);
    default: return qg::launch_gemm_nvf4_cluster_fits(c->tile_n, swap, c->stages, act_tiles);
  }
}

// Shared-memory and cluster feasibility of a launch (fused or not).
qg_status check_launch_fit(qg_format f, int M, int K, const qg_config* c, bool fused) {
  // covers the Block_FP8 scale columns and the activation slice as well
  if (gemm_smem(f, M, K, c, fused) > kSmemLimit) return QG_ERR_UNSUPPORTED;
  if (c->split_k > 1 && c->reduce_mode == qg::kReduceCluster &&
      (c->split_k > qg::kMaxClusterSplit || !cluster_fits(f, M, K, c, fused)))
    return QG_ERR_UNSUPPORTED;
  return QG_OK;
}

// The decode ("skinny") kernel: warp-level MMAs, no split-K; the eight
// compute warps form 64 / rows K groups (128 / rows for tile_n = 8) that take
// every K-group-th K tile, so the ring depth is a multiple of that.
qg_status check_skinny_config(qg_format f, const qg_config* c) {
  if (f == QG_NVFP4) return QG_ERR_UNSUPPORTED;
  if (c->split_k != 1 || c->swap_ab != 1 || c->reduce_mode != 0) return QG_ERR_UNSUPPORTED;
  if (c->tile_n != 8 && c->tile_n != 16 && c->tile_n != 32) return QG_ERR_UNSUPPORTED;
  if (c->rows != 8 && c->rows != 16 && c->rows != 32 && c->rows != 64) return QG_ERR_UNSUPPORTED;
  // tile_n = 8: a warp owns 16 weight rows (weights as the 16-row operand)
  if (c->tile_n == 8 && c->rows < 16) return QG_ERR_UNSUPPORTED;
  const int kg = (c->tile_n == 8 ? 128 : 64) / c->rows;
  if (c->stages < 2 || c->stages > 64 || c->stages % kg != 0) return QG_ERR_UNSUPPORTED;
  if (skinny_smem(f, c) > kSmemLimit) return QG_ERR_UNSUPPORTED;
  return QG_OK;
}

// The persistent kernel: the standard orientation without split-K, tiles of
// 128 or 256 channels, FP8_DYNAMIC, W8A8_INT8 and BLOCK_FP8 (bf16 output,
// checked at launch: the tile store needs a tensor map of y).
qg_status check_persist_config(qg_format f, int K, const qg_config* c) {
  if (f != QG_FP8_DYNAMIC && f != QG_W8A8_INT8 && f != QG_BLOCK_FP8) return QG_ERR_UNSUPPORTED;
  if (c->split_k != 1 || c->swap_ab != 0 || c->reduce_mode != 0 || c->rows != 0) return QG_ERR_UNSUPPORTED;
  if (c->tile_n != 128 && c->tile_n != 256) return QG_ERR_UNSUPPORTED;
  if (c->stages < 2 || c->stages > 12 || persist_smem(f, K, c) > kSmemLimit) return QG_ERR_UNSUPPORTED;
  return QG_OK;
}

// CTA pairs (variant 3): Block_FP8, standard orientation, 256 x tile_n
// pair tiles (tile_n 128 or 256), no split.
qg_status check_pair_config(qg_format f, int K, const qg_config* c) {
  if (f != QG_BLOCK_FP8) return QG_ERR_UNSUPPORTED;
  if (c->split_k != 1 || c->swap_ab != 0 || c->reduce_mode != 0 || c->rows != 0) return QG_ERR_UNSUPPORTED;
  if (c->tile_n != 128 && c->tile_n != 256) return QG_ERR_UNSUPPORTED;
  if (c->stages < 2 || c->stages > 12 || pair_smem(f, K, c) > kSmemLimit) return QG_ERR_UNSUPPORTED;
  return QG_OK;
}

qg_status check_config(qg_format f, int M, int N, int K, const qg_config* c) {
  if (!c) return QG_ERR_INVALID_ARG;
  if (c->reserved) return QG_ERR_INVALID_ARG;
  if (c->variant < 0 || c->variant > 3) return QG_ERR_INVALID_ARG;
  if (c->variant == 1) return check_skinny_config(f, c);
  if (c->variant == 2) return check_persist_config(f, K, c);
  if (c->variant == 3) return check_pair_config(f, K, c);
  if (c->rows != 0) return QG_ERR_INVALID_ARG;
  if (!is_pow2(c->split_k) || c->split_k > 256) return QG_ERR_UNSUPPORTED;
  if (c->swap_ab != 0 && c->swap_ab != 1) return QG_ERR_INVALID_ARG;
  if (c->reduce_mode < 0 || c->reduce_mode > 2) return QG_ERR_INVALID_ARG;
  const int tn = c->tile_n;
  if (tn != 16 && tn != 32 && tn != 64 && tn != 128 && tn != 256) return QG_ERR_UNSUPPORTED;
  // NVFP4 block scales of the N operand sit in TMEM words of 32 rows, and the
  // scale address an MMA takes must be an even word: a tile narrower than 64
  // rows must be the only tile (a 16-row tile at row 16, or a 32-row tile at
  // row 32, would start inside a word or at an odd one).
  if (f == QG_NVFP4 && tn < 64 && (c->swap_ab ? M : N) > tn) return QG_ERR_UNSUPPORTED;
  if (c->stages < 2 || c->stages > 12) return QG_ERR_UNSUPPORTED;
  const int kt = kt_total(f, K);
  if (c->split_k > kt) return QG_ERR_UNSUPPORTED;
  return check_launch_fit(f, M, K, c, false);
}

size_t ws_partial_bytes(int M, int N, int split) {
  return split > 1 ? align_up((size_t)split * M * N * 4, 256) : 0;
}
void tiles_of(const qg_config* c, int M, int N, int* tp, int* tq) {
  const int rows_p = c->swap_ab ? N : M;
  const int rows_q = c->swap_ab ? M : N;
  *tp = (rows_p + 127) / 128;
  *tq = (rows_q + c->tile_n - 1) / c->tile_n;
}

}  // namespace

extern "C" {

int qgemm_abi_version(void) { return QGEMM_ABI_VERSION; }

void qgemm_set_pdl(int enable) { g_pdl = enable != 0; }
void qgemm_set_tma_store(int enable) { g_tma_store = enable != 0; }

void qgemm_set_trace(void* device_buffer, size_t bytes) {
  g_trace = static_cast<unsigned long long*>(device_buffer);
  g_trace_bytes = device_buffer ? bytes : 0;
}

const char* qgemm_status_string(qg_status s) {
  switch (s) {
    case QG_OK: return "ok";
    case QG_ERR_INVALID_ARG: return "invalid argument";
    case QG_ERR_UNSUPPORTED: return "unsupported shape, configuration or device";
    case QG_ERR_WORKSPACE: return "workspace missing or too small";
    case QG_ERR_TABLE_IO: return "table file missing, corrupt or of another version";
    case QG_ERR_TABLE_MISS: return "no table entry";
    case QG_ERR_CUDA: return "CUDA error";
    case QG_ERR_DEVICE_TIMEOUT: return "in-kernel wait timed out";
    case QG_ERR_NO_DEVICE: return "no CUDA device";
  }
  return "unknown status";
}

qg_status qgemm_operand_bytes(qg_format f, int is_weight, int rows, int K, size_t* q_bytes,
                              size_t* scale_bytes) {
  if (!valid_format(f) || rows <= 0 || K <= 0 || !q_bytes || !scale_bytes) return QG_ERR_INVALID_ARG;
  if (K % k_multiple(f) != 0) return QG_ERR_INVALID_ARG;
  *q_bytes = (size_t)rows * row_bytes(f, K);
  switch (f) {
    case QG_FP8_DYNAMIC:
    case QG_W8A8_INT8: *scale_bytes = (size_t)rows * 4; break;
    case QG_BLOCK_FP8:
      *scale_bytes = (is_weight ? (size_t)((rows + 127) / 128) : (size_t)rows) * (K / 128) * 4;
      break;
    case QG_NVFP4:
      *scale_bytes = (size_t)((rows + 127) / 128) * 128 * (size_t)(((K + 255) / 256) * 16);
      break;
  }
  return QG_OK;
}

size_t qgemm_quant_workspace_size(qg_format f, int rows, int K) {
  (void)rows;
  (void)K;
  return f == QG_NVFP4 ? (size_t)qg::kNvfp4AmaxMaxCtas * 4 : 0;
}

size_t qgemm_workspace_size(qg_format f, int M, int N, int K, const qg_config* cfg) {
  if (!valid_format(f) || !cfg || M <= 0 || N <= 0 || K <= 0 || cfg->split_k <= 1) return 0;
  if (cfg->reduce_mode == qg::kReduceCluster) return 0;
  if (cfg->reduce_mode == qg::kReduceSecondPass) return ws_partial_bytes(M, N, cfg->split_k);
  int tp, tq;
  tiles_of(cfg, M, N, &tp, &tq);
  return ws_partial_bytes(M, N, cfg->split_k) + align_up((size_t)tp * tq * 4, 256);
}

qg_status qgemm_workspace_clear(void* workspace, size_t ws_bytes, void* stream) {
  if (ws_bytes == 0) return QG_OK;
  if (!workspace) return QG_ERR_INVALID_ARG;
  return cudaMemsetAsync(workspace, 0, ws_bytes, (cudaStream_t)stream) == cudaSuccess ? QG_OK
                                                                                     : QG_ERR_CUDA;
}

static qg_status check_quant_out(qg_format f, int rows, int K, const qg_operand* out) {
  if (!out || !out->q || !out->scale) return QG_ERR_INVALID_ARG;
  if (out->rows != rows || out->K != K) return QG_ERR_INVALID_ARG;
  if (!aligned(out->q, 16) || !aligned(out->scale, f == QG_NVFP4 ? 16 : 4)) return QG_ERR_INVALID_ARG;
  if (f == QG_NVFP4 && (!out->global_scale || !aligned(out->global_scale, 4))) return QG_ERR_INVALID_ARG;
  return QG_OK;
}

qg_status qgemm_quantize_act(qg_format f, const void* A, int M, int K, int lda,
                             const float* static_amax, qg_operand* out, void* workspace,
                             size_t ws_bytes, void* stream) {
  if (!valid_format(f) || !A || M <= 0 || K <= 0 || lda < K) return QG_ERR_INVALID_ARG;
  if (K % k_multiple(f) != 0 || (lda * 2) % 16 != 0 || !aligned(A, 16)) return QG_ERR_INVALID_ARG;
  qg_status s = check_quant_out(f, M, K, out);
  if (s != QG_OK) return s;
  const size_t need = qgemm_quant_workspace_size(f, M, K);
  if (f == QG_NVFP4 && static_amax == nullptr && (ws_bytes < need || !workspace))
    return QG_ERR_WORKSPACE;
  DeviceInfo* d;
  if ((s = device_info(&d)) != QG_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  switch (f) {
    case QG_FP8_DYNAMIC:
    case QG_W8A8_INT8:
      e = qg::launch_quant_rows(f == QG_W8A8_INT8, A, M, K, lda, out->q, (float*)out->scale, st, g_pdl);
      break;
    case QG_BLOCK_FP8:
      e = qg::launch_quant_act_groups(A, M, K, lda, out->q, (float*)out->scale, st, g_pdl);
      break;
    default:
      e = qg::launch_quant_nvfp4(A, M, K, lda, static_amax, out->q, out->scale, out->global_scale,
                                 (float*)workspace, st, g_pdl);
  }
  return e == cudaSuccess ? QG_OK : QG_ERR_CUDA;
}

qg_status qgemm_grouped_act_bytes(qg_format f, int experts, int T, int K, size_t* q_bytes,
                                  size_t* scale_bytes) {
  if (experts <= 0) return QG_ERR_INVALID_ARG;
  if (experts > qg::kMaxExperts) return QG_ERR_UNSUPPORTED;
  qg_status s = qgemm_operand_bytes(f, 0, T, K, q_bytes, scale_bytes);
  if (s != QG_OK || f != QG_NVFP4) return s;
  // every active expert (at most a = min(experts, T)) opens a fresh 128-row
  // atom: sum_e ceil(c_e / 128) <= floor((T - a) / 128) + a
  const int a = std::min(experts, T);
  *scale_bytes = (size_t)((T - a) / 128 + a) * 128 * (size_t)(((K + 255) / 256) * 16);
  return QG_OK;
}

qg_status qgemm_quantize_act_grouped(qg_format f, int experts, const int* expert_offsets, const void* A,
                                     int T, int K, int lda, const float* static_amax, qg_operand* out,
                                     void* workspace, size_t ws_bytes, void* stream) {
  if (experts <= 0 || !expert_offsets || !aligned(expert_offsets, 4)) return QG_ERR_INVALID_ARG;
  if (experts > qg::kMaxExperts) return QG_ERR_UNSUPPORTED;
  // the 8-bit formats' scales are per token (group): their layout does not
  // depend on the routing
  if (f != QG_NVFP4) return qgemm_quantize_act(f, A, T, K, lda, static_amax, out, workspace, ws_bytes, stream);
  if (!A || T <= 0 || K <= 0 || lda < K) return QG_ERR_INVALID_ARG;
  if (K % k_multiple(f) != 0 || (lda * 2) % 16 != 0 || !aligned(A, 16)) return QG_ERR_INVALID_ARG;
  qg_status s = check_quant_out(f, T, K, out);
  if (s != QG_OK) return s;
  if (static_amax == nullptr && (ws_bytes < qgemm_quant_workspace_size(f, T, K) || !workspace))
    return QG_ERR_WORKSPACE;
  DeviceInfo* d;
  if ((s = device_info(&d)) != QG_OK) return s;
  const cudaError_t e = qg::launch_quant_nvfp4(A, T, K, lda, static_amax, out->q, out->scale, out->global_scale,
                                               (float*)workspace, (cudaStream_t)stream, g_pdl, expert_offsets,
                                               experts);
  return e == cudaSuccess ? QG_OK : QG_ERR_CUDA;
}

qg_status qgemm_quantize_weight(qg_format f, const void* W, int N, int K, qg_operand* out,
                                void* workspace, size_t ws_bytes, void* stream) {
  if (!valid_format(f) || !W || N <= 0 || K <= 0) return QG_ERR_INVALID_ARG;
  if (K % k_multiple(f) != 0 || !aligned(W, 16)) return QG_ERR_INVALID_ARG;
  qg_status s = check_quant_out(f, N, K, out);
  if (s != QG_OK) return s;
  if (f == QG_NVFP4 && (ws_bytes < qgemm_quant_workspace_size(f, N, K) || !workspace))
    return QG_ERR_WORKSPACE;
  DeviceInfo* d;
  if ((s = device_info(&d)) != QG_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  switch (f) {
    case QG_FP8_DYNAMIC:
    case QG_W8A8_INT8:
      e = qg::launch_quant_rows(f == QG_W8A8_INT8, W, N, K, K, out->q, (float*)out->scale, st, g_pdl);
      break;
    case QG_BLOCK_FP8:
      e = qg::launch_quant_weight_blocks(W, N, K, out->q, (float*)out->scale, st, g_pdl);
      break;
    default:
      e = qg::launch_quant_nvfp4(W, N, K, K, nullptr, out->q, out->scale, out->global_scale,
                                 (float*)workspace, st, g_pdl);
  }
  return e == cudaSuccess ? QG_OK : QG_ERR_CUDA;
}

qg_status qgemm_quantize_weight_grouped(qg_format f, int experts, const void* W, int N, int K,
                                        qg_operand* out, void* workspace, size_t ws_bytes, void* stream) {
  if (experts <= 0 || N <= 0 || N % 128 != 0 || !out) return QG_ERR_INVALID_ARG;
  if (experts > qg::kMaxExperts) return QG_ERR_UNSUPPORTED;
  if ((long long)experts * N > 0x7fffffffLL) return QG_ERR_INVALID_ARG;
  // per-row and 128x128-block scales never cross an expert boundary
  // (N % 128 == 0): the stacked tensor quantises as each expert would
  if (f != QG_NVFP4) return qgemm_quantize_weight(f, W, experts * N, K, out, workspace, ws_bytes, stream);
  if (!W || K <= 0 || K % k_multiple(f) != 0 || !aligned(W, 16)) return QG_ERR_INVALID_ARG;
  qg_status s = check_quant_out(f, experts * N, K, out);
  if (s != QG_OK) return s;
  if (ws_bytes < qgemm_quant_workspace_size(f, N, K) || !workspace) return QG_ERR_WORKSPACE;
  DeviceInfo* d;
  if ((s = device_info(&d)) != QG_OK) return s;
  // NVFP4: each expert is its own tensor with its own tensor scale; its
  // codes, block scales (whole 128-row atoms) and tensor scale sit at
  // expert x (N rows) in the stacked buffers
  size_t qb = 0, sb = 0;
  if ((s = qgemm_operand_bytes(f, 1, N, K, &qb, &sb)) != QG_OK) return s;
  const __nv_bfloat16* w = static_cast<const __nv_bfloat16*>(W);
  for (int e = 0; e < experts; ++e) {
    const cudaError_t err = qg::launch_quant_nvfp4(
        w + (size_t)e * N * K, N, K, K, nullptr, static_cast<uint8_t*>(out->q) + (size_t)e * qb,
        static_cast<uint8_t*>(out->scale) + (size_t)e * sb, out->global_scale + e, (float*)workspace,
        (cudaStream_t)stream, g_pdl);
    if (err != cudaSuccess) return QG_ERR_CUDA;
  }
  return QG_OK;
}

qg_status check_operand_impl(qg_format f, const qg_operand* o, int rows, int K) {
  if (!o || !o->q || !o->scale) return QG_ERR_INVALID_ARG;
  if (o->rows != rows || o->K != K) return QG_ERR_INVALID_ARG;
  if (!aligned(o->q, 16) || !aligned(o->scale, f == QG_NVFP4 ? 16 : 4)) return QG_ERR_INVALID_ARG;
  if (f == QG_NVFP4 && (!o->global_scale || !aligned(o->global_scale, 4))) return QG_ERR_INVALID_ARG;
  return QG_OK;
}

}  // extern "C"

namespace qg {
// Host-side argument checks of qgemm_run (no device work).
qg_status check_run_args(qg_format f, const qg_operand* A, const qg_operand* W, int M, int N, int K,
                         const qg_config* cfg, void* workspace, size_t ws_bytes, void* Y, int ldy,
                         int out_kind) {
  if (!valid_format(f) || M <= 0 || N <= 0 || K <= 0 || !Y || ldy < N) return QG_ERR_INVALID_ARG;
  if (out_kind != QG_OUT_BF16 && out_kind != QG_OUT_ACC) return QG_ERR_INVALID_ARG;
  if (K % k_multiple(f) != 0 || !aligned(Y, 16)) return QG_ERR_INVALID_ARG;
  qg_status s;
  if ((s = check_operand_impl(f, A, M, K)) != QG_OK) return s;
  if ((s = check_operand_impl(f, W, N, K)) != QG_OK) return s;
  if ((s = check_config(f, M, N, K, cfg)) != QG_OK) return s;
  const size_t need = qgemm_workspace_size(f, M, N, K, cfg);
  if (need > 0 && (!workspace || ws_bytes < need || !aligned(workspace, 256))) return QG_ERR_WORKSPACE;
  return QG_OK;
}

// Host-side argument checks of qgemm_run_fused_act (no device work).
qg_status check_fused_args(qg_format f, const void* A, int lda, const qg_operand* W, int M, int N, int K,
                           const qg_config* cfg, void* workspace, size_t ws_bytes, void* Y, int ldy,
                           int out_kind, const float* act_scale_out) {
  if (!valid_format(f) || M <= 0 || N <= 0 || K <= 0 || !Y || ldy < N || !A || lda < K)
    return QG_ERR_INVALID_ARG;
  if (out_kind != QG_OUT_BF16 && out_kind != QG_OUT_ACC) return QG_ERR_INVALID_ARG;
  if (K % k_multiple(f) != 0 || !aligned(Y, 16) || !aligned(A, 16) || (lda * 2) % 16 != 0)
    return QG_ERR_INVALID_ARG;
  if (act_scale_out != nullptr && !aligned(act_scale_out, 4)) return QG_ERR_INVALID_ARG;
  // NVFP4's tensor scale needs the amax of the whole activation tensor
  if (f == QG_NVFP4) return QG_ERR_UNSUPPORTED;
  qg_status s;
  if ((s = check_operand_impl(f, W, N, K)) != QG_OK) return s;
  if ((s = check_config(f, M, N, K, cfg)) != QG_OK) return s;
  if (cfg->swap_ab != 1 || cfg->variant != 0) return QG_ERR_UNSUPPORTED;
  // the whole activation slice of a CTA is held in shared memory
  if ((s = check_launch_fit(f, M, K, cfg, true)) != QG_OK) return s;
  // a per-token scale spans all of K: split-K slices must meet in a cluster
  if (f != QG_BLOCK_FP8 && cfg->split_k > 1 && cfg->reduce_mode != kReduceCluster)
    return QG_ERR_UNSUPPORTED;
  const size_t need = qgemm_workspace_size(f, M, N, K, cfg);
  if (need > 0 && (!workspace || ws_bytes < need || !aligned(workspace, 256))) return QG_ERR_WORKSPACE;
  return QG_OK;
}
}  // namespace qg

namespace {
// Launch of the GEMM (and, for reduce_mode 1, its second pass) after the
// arguments were checked.  `A` is the quantised activation operand, or null
// when the kernel quantises the bf16 activations `act` itself (fused).
qg_status launch_run(qg_format f, const qg_operand* A, const void* act, int lda, float* act_scale_out,
                     const qg_operand* W, int M, int N, int K, const qg_config* cfg, void* workspace,
                     void* Y, int ldy, int out_kind, void* stream, int experts = 0,
                     const int* expert_offsets = nullptr) {
  DeviceInfo* d;
  qg_status s;
  if ((s = device_info(&d)) != QG_OK) return s;

  const bool swap = cfg->swap_ab != 0;
  GemmParams prm = {};
  prm.M = M;
  prm.N = N;
  prm.K = K;
  prm.rows_p = swap ? N : M;
  prm.rows_q = swap ? M : N;
  prm.kt_total = kt_total(f, K);
  prm.split_k = cfg->split_k;
  prm.stages = cfg->stages;
  prm.groups = K / 128;
  prm.scale_a = A ? static_cast<const float*>(A->scale) : nullptr;
  prm.scale_w = static_cast<const float*>(W->scale);
  const uint8_t* sfa = A ? static_cast<const uint8_t*>(A->scale) : nullptr;
  const uint8_t* sfw = static_cast<const uint8_t*>(W->scale);
  prm.sf_p = swap ? sfw : sfa;
  prm.sf_q = swap ? sfa : sfw;
  prm.sf_atoms_per_rb = ((K + 255) / 256) * 4;
  prm.g_a = A ? A->global_scale : nullptr;
  prm.g_w = W->global_scale;
  prm.Y = Y;
  prm.ldy = ldy;
  prm.out_kind = out_kind;
  prm.act = static_cast<const __nv_bfloat16*>(act);
  prm.lda = lda;
  prm.act_scale_out = act_scale_out;
  int tp, tq;
  tiles_of(cfg, M, N, &tp, &tq);
  if (cfg->variant == 2) {
    // persistent kernel: one CTA per SM (at most the tiles) walking the
    // output tiles; the tile store needs bf16 output through a tensor map of y
    if (out_kind != QG_OUT_BF16 || act != nullptr || expert_offsets != nullptr) return QG_ERR_UNSUPPORTED;
    prm.nkt_max = prm.kt_total;
    prm.err = d->err;
    prm.wait_ns = g_wait_ns;
    const long long tiles = (long long)((M + 127) / 128) * ((N + cfg->tile_n - 1) / cfg->tile_n);
    const int ctas = (int)std::min<long long>(tiles, d->sms > 0 ? d->sms : 148);
    if (g_trace != nullptr && (size_t)ctas * qg::kTraceEvents * sizeof(unsigned long long) <= g_trace_bytes)
      prm.trace = g_trace;
    CUtensorMap tp, tq, ty;
    const uint64_t rb = row_bytes(f, K);
    if (!make_tmap(&tp, A->q, rb, (uint64_t)M, 128)) return QG_ERR_CUDA;
    if (!make_tmap(&tq, W->q, rb, (uint64_t)N, (uint32_t)cfg->tile_n)) return QG_ERR_CUDA;
    if (!make_tmap_y(&ty, Y, N, M, ldy)) return QG_ERR_UNSUPPORTED;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e;
    switch (f) {
      case QG_FP8_DYNAMIC: e = qg::launch_gemm_fp8_persist(cfg->tile_n, tp, tq, ty, prm, dim3(ctas), st, g_pdl); break;
      case QG_W8A8_INT8: e = qg::launch_gemm_int8_persist(cfg->tile_n, tp, tq, ty, prm, dim3(ctas), st, g_pdl); break;
      default: e = qg::launch_gemm_block_persist(cfg->tile_n, tp, tq, ty, prm, dim3(ctas), st, g_pdl); break;
    }
    if (e != cudaSuccess) return e == cudaErrorInvalidValue ? QG_ERR_UNSUPPORTED : QG_ERR_CUDA;
    return QG_OK;
  }
  if (cfg->variant == 3) {
    // CTA pairs: clusters of two CTAs (one per SM) walking the 256 x tile_n
    // output tiles; bf16 output through a tensor map of y
    if (out_kind != QG_OUT_BF16 || act != nullptr || expert_offsets != nullptr) return QG_ERR_UNSUPPORTED;
    prm.nkt_max = prm.kt_total;
    prm.err = d->err;
    prm.wait_ns = g_wait_ns;
    const long long tiles = (long long)((M + 255) / 256) * ((N + cfg->tile_n - 1) / cfg->tile_n);
    const int pairs = (int)std::min<long long>(tiles, (d->sms > 0 ? d->sms : 148) / 2);
    const int ctas = 2 * pairs;
    if (g_trace != nullptr && (size_t)ctas * qg::kTraceEvents * sizeof(unsigned long long) <= g_trace_bytes)
      prm.trace = g_trace;
    CUtensorMap tp, tq, ty;
    const uint64_t rb = row_bytes(f, K);
    if (!make_tmap(&tp, A->q, rb, (uint64_t)M, 128)) return QG_ERR_CUDA;
    if (!make_tmap(&tq, W->q, rb, (uint64_t)N, (uint32_t)(cfg->tile_n / 2))) return QG_ERR_CUDA;
    if (!make_tmap_y(&ty, Y, N, M, ldy)) return QG_ERR_UNSUPPORTED;
    const cudaError_t e =
        qg::launch_gemm_block_pair(cfg->tile_n, tp, tq, ty, prm, dim3(ctas), (cudaStream_t)stream, g_pdl);
    if (e != cudaSuccess) return e == cudaErrorInvalidValue ? QG_ERR_UNSUPPORTED : QG_ERR_CUDA;
    return QG_OK;
  }
  if (cfg->variant == 1) {
    // decode kernel: CTA (x, y) = weight rows [x rows, (x + 1) rows) x
    // tokens [y tile_n, (y + 1) tile_n), the whole of K
    prm.nkt_max = prm.kt_total;
    prm.err = d->err;
    prm.wait_ns = g_wait_ns;
    const int gx = (N + cfg->rows - 1) / cfg->rows, gy = (M + cfg->tile_n - 1) / cfg->tile_n;
    if (gy > 65535) return QG_ERR_UNSUPPORTED;
    if (g_trace != nullptr &&
        (size_t)gx * gy * qg::kTraceEvents * sizeof(unsigned long long) <= g_trace_bytes)
      prm.trace = g_trace;
    if (g_l2_ahead) prm.l2_ahead = (gx * gy + 1) / 2;
    CUtensorMap tw, ta;
    const uint64_t rb = row_bytes(f, K);
    if (!make_tmap(&tw, W->q, rb, (uint64_t)N, (uint32_t)cfg->rows)) return QG_ERR_CUDA;
    if (!make_tmap(&ta, A->q, rb, (uint64_t)M, (uint32_t)cfg->tile_n)) return QG_ERR_CUDA;
    const dim3 grid(gx, gy, 1);
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e;
    switch (f) {
      case QG_FP8_DYNAMIC: e = qg::launch_gemm_fp8_skinny(cfg->tile_n, cfg->rows, tw, ta, prm, grid, st, g_pdl); break;
      case QG_W8A8_INT8: e = qg::launch_gemm_int8_skinny(cfg->tile_n, cfg->rows, tw, ta, prm, grid, st, g_pdl); break;
      case QG_BLOCK_FP8: e = qg::launch_gemm_block_skinny(cfg->tile_n, cfg->rows, tw, ta, prm, grid, st, g_pdl); break;
      default: return QG_ERR_UNSUPPORTED;
    }
    if (e != cudaSuccess) return e == cudaErrorInvalidValue ? QG_ERR_UNSUPPORTED : QG_ERR_CUDA;
    return QG_OK;
  }
  if (cfg->split_k > 1 && cfg->reduce_mode != qg::kReduceCluster) {
    prm.partial = workspace;
    prm.counters = reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(workspace) +
                                                   ws_partial_bytes(M, N, cfg->split_k));
  }
  prm.reduce_mode = cfg->reduce_mode;
  const LaunchShape ls = launch_shape(f, M, K, cfg, act != nullptr);
  prm.nkt_max = ls.nkt_max;
  prm.recv_cols = ls.recv_cols;
  prm.a_mode = ls.a_mode;
  prm.experts = experts;
  prm.expert_offsets = expert_offsets;
  prm.err = d->err;
  prm.wait_ns = g_wait_ns;
  if (g_trace != nullptr &&
      (size_t)tp * tq * cfg->split_k * qg::kTraceEvents * sizeof(unsigned long long) <= g_trace_bytes)
    prm.trace = g_trace;

  CUtensorMap tmp, tmq, tmy;
  std::memset(&tmy, 0, sizeof(tmy));
  // direct standard-orientation tiles of 64 channels or more store bf16
  // through a tensor map of y (a map that does not encode, e.g. for an
  // unaligned y, leaves the thread stores)
  prm.y_tma = 0;
  if (g_tma_store && !swap && out_kind == 0 && cfg->split_k == 1 && cfg->tile_n >= 64 && act == nullptr &&
      expert_offsets == nullptr && make_tmap_y(&tmy, Y, N, M, ldy))
    prm.y_tma = 1;
  const uint64_t rb = row_bytes(f, K);
  // grouped: the P tensor is every expert's weight rows, [experts * N, K]
  const uint64_t p_rows = expert_offsets ? (uint64_t)experts * N : (uint64_t)prm.rows_p;
  if (!make_tmap(&tmp, swap ? W->q : A->q, rb, p_rows, 128)) return QG_ERR_CUDA;
  if (A != nullptr) {
    if (!make_tmap(&tmq, swap ? A->q : W->q, rb, (uint64_t)prm.rows_q, (uint32_t)cfg->tile_n))
      return QG_ERR_CUDA;
  } else {
    tmq = tmp;                                 // fused: the kernel writes the Q tiles itself
  }
  // grouped: one y index per token tile of any expert.  An expert with c > 0
  // tokens has ceil(c / tile_n) <= (c - 1) / tile_n + 1 tiles; over at most
  // a = min(experts, M) such experts that sums to at most
  // floor((M - a) / tile_n) + a (nondecreasing in the number of experts), so
  // the grid needs no routing from the host.  CTAs past the last tile exit,
  // and each costs launch and retire time, so the bound is kept tight.
  if (expert_offsets) {
    const int a = std::min(experts, M);
    tq = (M - a) / cfg->tile_n + a;
  }
  if (tq > 65535) return QG_ERR_UNSUPPORTED;
  const dim3 grid(tp, tq, cfg->split_k);
  // weight prefetch for the later half of a Swap-AB grid (launch order:
  // clusters of split_k, else single CTAs); not for grouped launches, whose
  // weight rows depend on the routing
  // (the kernel indexes the grid in 32 bits: only grids below 2^31 CTAs)
  if (swap && !expert_offsets && act == nullptr && g_l2_ahead &&
      (long long)tp * tq * cfg->split_k < 0x7fffffffLL) {
    const bool clus = cfg->split_k > 1 && cfg->reduce_mode == qg::kReduceCluster;
    const long long units = clus ? (long long)tp * tq : (long long)tp * tq * cfg->split_k;
    prm.l2_ahead = (int)((units + 1) / 2);
  }
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  switch (f) {
    case QG_FP8_DYNAMIC: e = qg::launch_gemm_fp8(swap, cfg->tile_n, tmp, tmq, tmy, prm, grid, st, g_pdl); break;
    case QG_W8A8_INT8: e = qg::launch_gemm_int8(swap, cfg->tile_n, tmp, tmq, tmy, prm, grid, st, g_pdl); break;
    case QG_BLOCK_FP8: e = qg::launch_gemm_block(swap, cfg->tile_n, tmp, tmq, tmy, prm, grid, st, g_pdl); break;
    default: e = qg::launch_gemm_nvf4(swap, cfg->tile_n, tmp, tmq, tmy, prm, grid, st, g_pdl); break;
  }
  if (e != cudaSuccess) return e == cudaErrorInvalidValue ? QG_ERR_UNSUPPORTED : QG_ERR_CUDA;
  if (cfg->split_k > 1 && cfg->reduce_mode == qg::kReduceSecondPass) {
    switch (f) {
      case QG_FP8_DYNAMIC: e = qg::launch_gemm_fp8_reduce(prm, st, g_pdl); break;
      case QG_W8A8_INT8: e = qg::launch_gemm_int8_reduce(prm, st, g_pdl); break;
      case QG_BLOCK_FP8: e = qg::launch_gemm_block_reduce(prm, st, g_pdl); break;
      default: e = qg::launch_gemm_nvf4_reduce(prm, st, g_pdl); break;
    }
    if (e != cudaSuccess) return QG_ERR_CUDA;
  }
  return QG_OK;
}
}  // namespace

extern "C" {

qg_status qgemm_run(qg_format f, const qg_operand* A, const qg_operand* W, int M, int N, int K,
                    const qg_config* cfg, void* workspace, size_t ws_bytes, void* Y, int ldy,
                    int out_kind, void* stream) {
  qg_status s = qg::check_run_args(f, A, W, M, N, K, cfg, workspace, ws_bytes, Y, ldy, out_kind);
  if (s != QG_OK) return s;
  return launch_run(f, A, nullptr, 0, nullptr, W, M, N, K, cfg, workspace, Y, ldy, out_kind, stream);
}

qg_status qgemm_run_grouped(qg_format f, int experts, const int* expert_offsets, const qg_operand* A,
                            const qg_operand* W, int N, int K, const qg_config* cfg, void* workspace,
                            size_t ws_bytes, void* Y, int ldy, int out_kind, void* stream) {
  if (!valid_format(f) || experts <= 0 || !expert_offsets || !A || !W || !aligned(expert_offsets, 4))
    return QG_ERR_INVALID_ARG;
  if (experts > qg::kMaxExperts) return QG_ERR_UNSUPPORTED;
  if (N <= 0 || N % 128 != 0) return QG_ERR_INVALID_ARG;   // experts' weight rows fill whole 128-row blocks
  if ((long long)experts * N > 0x7fffffffLL) return QG_ERR_INVALID_ARG;
  const int M = A->rows;
  qg_operand Wall = *W;                                    // the operand checks see one expert's rows
  if (W->rows != experts * N) return QG_ERR_INVALID_ARG;
  Wall.rows = N;
  qg_status s = qg::check_run_args(f, A, &Wall, M, N, K, cfg, workspace, ws_bytes, Y, ldy, out_kind);
  if (s != QG_OK) return s;
  if (cfg->swap_ab != 1 || cfg->variant != 0) return QG_ERR_UNSUPPORTED;
  if (cfg->split_k > 1 && cfg->reduce_mode == qg::kReduceLastCta) return QG_ERR_UNSUPPORTED;
  return launch_run(f, A, nullptr, 0, nullptr, W, M, N, K, cfg, workspace, Y, ldy, out_kind, stream, experts,
                    expert_offsets);
}

qg_status qgemm_run_fused_act(qg_format f, const void* A, int lda, const qg_operand* W, int M, int N,
                              int K, const qg_config* cfg, void* workspace, size_t ws_bytes, void* Y,
                              int ldy, int out_kind, float* act_scale_out, void* stream) {
  qg_status s = qg::check_fused_args(f, A, lda, W, M, N, K, cfg, workspace, ws_bytes, Y, ldy, out_kind,
                                     act_scale_out);
  if (s != QG_OK) return s;
  return launch_run(f, nullptr, A, lda, act_scale_out, W, M, N, K, cfg, workspace, Y, ldy, out_kind,
                    stream);
}

qg_status qgemm_default_config(qg_format f, int M, int N, int K, qg_config* out) {
  if (!valid_format(f) || M <= 0 || N <= 0 || K <= 0 || !out) return QG_ERR_INVALID_ARG;
  if (K % k_multiple(f) != 0) return QG_ERR_INVALID_ARG;
  // the analytic scorer's best-ranked configuration; the fixed rule below
  // only if no candidate of the scorer's grid is feasible
  int n = 0;
  if (qgemm_rank_configs(f, M, N, K, out, 1, nullptr, &n) == QG_OK && n == 1) return QG_OK;
  return qg::rule_default_config(f, M, N, K, out);
}

qg_status qgemm_grouped_default_config(qg_format f, int experts, int T, int N, int K, qg_config* out) {
  if (!valid_format(f) || experts <= 0 || T <= 0 || N <= 0 || K <= 0 || !out) return QG_ERR_INVALID_ARG;
  if (K % k_multiple(f) != 0) return QG_ERR_INVALID_ARG;
  // T tokens over at most min(experts, T) experts: the launch streams the
  // weights of the active experts, like one GEMM of active x N rows with the
  // mean token count per expert
  const int active = std::min(experts, T);
  const int m_eff = (T + active - 1) / active;
  const long long rows = (long long)active * N;
  if (rows <= (long long)INT32_MAX) {
    qg_config ranked[256];
    int n = 0;
    if (qgemm_rank_configs(f, m_eff, (int)rows, K, ranked, 256, nullptr, &n) == QG_OK)
      for (int i = 0; i < n; ++i)
        if (ranked[i].variant == 0 && ranked[i].swap_ab == 1 && ranked[i].reduce_mode != 2 &&
            qg::config_check(f, T, N, K, &ranked[i]) == QG_OK) {
          *out = ranked[i];
          return QG_OK;
        }
  }
  qg_config c = {};
  c.split_k = 1;
  c.swap_ab = 1;
  c.tile_n = (f == QG_NVFP4 && T > 16) ? 64 : 16;    // NVFP4: narrow tiles only as the sole tile
  c.stages = 4;
  if (qg::config_check(f, T, N, K, &c) != QG_OK) return QG_ERR_UNSUPPORTED;
  *out = c;
  return QG_OK;
}

}  // extern "C"

// Name (spaces as '_') and SM count of the current device, for the table's
// identity gate; false without a device.
bool qg_current_device(char* name, size_t cap, int* sms) {
  int dev = 0;
  cudaDeviceProp p;
  if (cap == 0 || cudaGetDevice(&dev) != cudaSuccess || cudaGetDeviceProperties(&p, dev) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  std::snprintf(name, cap, "%s", p.name);
  for (char* c = name; *c; ++c)
    if (*c == ' ') *c = '_';
  *sms = p.multiProcessorCount;
  return true;
}

namespace qg {
// Feasibility and shared memory of a configuration, for the scorer.
qg_status config_check(qg_format f, int M, int N, int K, const qg_config* c) {
  return check_config(f, M, N, K, c);
}
size_t config_smem(qg_format f, int M, int K, const qg_config* c) { return gemm_smem(f, M, K, c, false); }
int device_sm_count() {
  DeviceInfo* d;
  return device_info(&d) == QG_OK ? d->sms : 148;
}

// The fixed-rule default (before the analytic scorer): Swap-AB up to 64
// tokens, split-K filling the SMs, the deepest ring that fits.
qg_status rule_default_config(qg_format f, int M, int N, int K, qg_config* out) {
  qg_config c = {};
  c.reduce_mode = 0;
  // Swap-AB below 32 tokens (and up to 64, where tokens still fit the MMA N
  // slot in one tile); the standard orientation above.
  c.swap_ab = M <= 64 ? 1 : 0;
  if (c.swap_ab) {
    c.tile_n = M <= 16 ? 16 : M <= 32 ? 32 : 64;
  } else {
    c.tile_n = 256;
  }
  // split-K: fill the SMs with tiles x split, keeping >= 2 K tiles per split
  int tp, tq;
  c.split_k = 1;
  tiles_of(&c, M, N, &tp, &tq);
  const int tiles = tp * tq;
  const int kt = kt_total(f, K);
  int sms = 148;
  DeviceInfo* d;
  if (device_info(&d) == QG_OK) sms = d->sms;
  while (c.split_k < 256 && tiles * c.split_k * 2 <= sms && kt / (c.split_k * 2) >= 2) c.split_k *= 2;
  // deepest pipeline that fits, at most 8 stages; a Block_FP8 slice whose
  // scale columns leave no room for two stages is split further
  for (;;) {
    c.stages = 0;
    for (int s = 8; s >= 2; --s) {
      c.stages = s;
      if (gemm_smem(f, M, K, &c, false) <= kSmemLimit) break;
      c.stages = 0;
    }
    if (c.stages != 0) break;
    if (c.split_k >= 256 || c.split_k * 2 > kt) return QG_ERR_UNSUPPORTED;
    c.split_k *= 2;
  }
  // split-K partials meet in distributed shared memory when the cluster
  // fits, else the last-arriving CTA sums them from the workspace
  c.reduce_mode = (c.split_k <= qg::kMaxClusterSplit && cluster_fits(f, M, K, &c, false))
                      ? qg::kReduceCluster
                      : qg::kReduceLastCta;
  *out = c;
  return QG_OK;
}
}  // namespace qg

extern "C" {

void qgemm_set_wait_limit(unsigned long long limit_ns) {
  g_wait_ns = limit_ns > 0 ? limit_ns : qg::kWaitLimitNs;
}

qg_status qgemm_selftest_wait_expiry(unsigned long long limit_ns, void* stream) {
  if (limit_ns == 0 || limit_ns > qg::kWaitLimitNs) return QG_ERR_INVALID_ARG;
  DeviceInfo* d;
  qg_status s = device_info(&d);
  if (s != QG_OK) return s;
  wait_expiry_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(d->err, limit_ns);
  return cudaGetLastError() == cudaSuccess ? QG_OK : QG_ERR_CUDA;
}

qg_status qgemm_device_error(void) {
  DeviceInfo* d;
  qg_status s = device_info(&d);
  if (s != QG_OK) return s;
  if (cudaDeviceSynchronize() != cudaSuccess) return QG_ERR_CUDA;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, qg::g_qg_error, sizeof(v)) != cudaSuccess) return QG_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(qg::g_qg_error, &zero, sizeof(zero)) != cudaSuccess) return QG_ERR_CUDA;
  return v ? QG_ERR_DEVICE_TIMEOUT : QG_OK;
}

}  // extern "C"
