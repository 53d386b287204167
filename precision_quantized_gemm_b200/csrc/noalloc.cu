// noalloc.cu — qgemm_run_noalloc: qgemm_run for callers that cannot allocate.
//
// Split-K with reduce_mode 1 or 2 needs scratch memory for its partial sums
// (and, for mode 2, per-tile arrival counters).  qgemm_run takes that scratch
// from the caller.  Some callers cannot provide it: an inference engine whose
// memory planner reserved all device memory up front and forbids allocation
// while serving, a plugin host that hands a kernel library only its input and
// output buffers, or code that must not call cudaMalloc on this path at all.
// For them this entry point uses a fixed scratch array that lives in the
// library itself (a file-scope __device__ array, present on every GPU that
// loads the library until the process exits) and calls no allocator.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/qgemm.h"
#include "internal.h"

namespace {

constexpr size_t kScratchBytes = (size_t)QGEMM_NOALLOC_SCRATCH_BYTES;

// The scratch array.  In host code `g_noalloc_scratch` names a host-side
// stand-in, not device memory: its device address must come from
// cudaGetSymbolAddress (below), once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_mu;

// Device address of the scratch array on the current device, looked up on
// the first call per device with that device current.  That lookup may load
// the library's device code, which a stream being captured into a CUDA graph
// does not allow: a first call on a device made during capture is refused
// with QG_ERR_UNSUPPORTED (make one call before capturing), not attempted.
qg_status scratch_address(cudaStream_t stream, void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QG_ERR_NO_DEVICE;
  if (dev < 0 || dev >= kMaxDevices) return QG_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return QG_ERR_CUDA;
    if (cs != cudaStreamCaptureStatusNone) return QG_ERR_UNSUPPORTED;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return QG_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return QG_OK;
}

// A 256-byte aligned non-null stand-in that lets the argument checks accept
// the scratch before its device address is known (never dereferenced).
void* g_scratch_probe() { return reinterpret_cast<void*>(static_cast<uintptr_t>(256)); }

}  // namespace

extern "C" qg_status qgemm_run_noalloc(qg_format f, const qg_operand* A, const qg_operand* W, int M,
                                       int N, int K, const qg_config* cfg, void* Y, int ldy,
                                       int out_kind, void* stream) {
  if (!cfg) return QG_ERR_INVALID_ARG;
  const size_t need = qgemm_workspace_size(f, M, N, K, cfg);
  if (need > kScratchBytes) return QG_ERR_WORKSPACE;
  // every argument other than the scratch is checked before it is touched
  qg_status s0 = qg::check_run_args(f, A, W, M, N, K, cfg, need ? g_scratch_probe() : nullptr, need, Y,
                                    ldy, out_kind);
  if (s0 != QG_OK) return s0;
  void* scratch = nullptr;
  if (need > 0) {
    qg_status s = scratch_address((cudaStream_t)stream, &scratch);
    if (s != QG_OK) return s;
    // The array keeps the previous call's contents.  Partial sums are fully
    // rewritten before they are read; the tile counters of reduce_mode 2 must
    // start at zero, so that region is cleared here (a memset, not an
    // allocation).
    if (cfg->split_k > 1 && cfg->reduce_mode == 2) {
      const size_t partial = (((size_t)cfg->split_k * M * N * 4) + 255) / 256 * 256;
      if (cudaMemsetAsync(static_cast<unsigned char*>(scratch) + partial, 0, need - partial,
                          (cudaStream_t)stream) != cudaSuccess)
        return QG_ERR_CUDA;
    }
  }
  return qgemm_run(f, A, W, M, N, K, cfg, scratch, need, Y, ldy, out_kind, stream);
}
