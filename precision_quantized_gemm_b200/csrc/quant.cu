// quant.cu — dynamic activation quantisation and offline weight quantisation.
//
// The "quantization" auxiliary kernel of "Helion in the vLLM backend"
// (seventh paragraph), one pass per row / group with 16-byte vector loads:
//   amax -> scale = amax / Qmax (correctly rounded fp32 division) ->
//   code = round-to-nearest-even(x / scale), saturating to the format.
// All-zero rows, groups and tensors get scale 1 (and codes 0).
//   FP8_DYNAMIC  e4m3 per row (token or channel), Qmax 448
//   W8A8_INT8    int8 per row, Qmax 127, clamp to [-127, 127]
//   BLOCK_FP8    e4m3 per 1x128 activation group / 128x128 weight block
//   NVFP4        e2m1 per element, e4m3 scale per 16 elements, fp32 tensor
//                scale g = amax / (448 * 6); block scale e4m3((amax_b/6)/g);
//                code e2m1(x / (dec(block scale) * g)); block scales stored
//                in the 128x4 tiled layout the GEMM copies into TMEM.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "ptx.cuh"
#include "quant_math.cuh"

namespace qg {

namespace {

constexpr int kQThreads = 256;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ float block_max(float v, float* red) {
  v = warp_max(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  if (w == 0) {
    float t = (l < (int)(blockDim.x >> 5)) ? red[l] : 0.f;
    t = warp_max(t);
    if (l == 0) red[0] = t;
  }
  __syncthreads();
  return red[0];
}

// ---------------------------------------------- per-row e4m3 / int8 rows --
// One CTA per row; up to 4 chunks of 8 elements per thread stay in registers
// between the amax and the quantisation pass.
template <bool INT8>
__global__ void __launch_bounds__(kQThreads) quant_rows_kernel(const __nv_bfloat16* __restrict__ X,
                                                               int K, int ldx, uint8_t* __restrict__ q,
                                                               float* __restrict__ scale) {
  __shared__ float red[32];
  // let the next kernel (the GEMM) start streaming its weights now; it
  // waits for this kernel's completion before it reads what we write
  griddep_launch_dependents();
  griddep_wait();
  const int r = blockIdx.x;
  const uint4* row = reinterpret_cast<const uint4*>(X + (size_t)r * ldx);
  const int nch = K / 8;
  uint4 cache[4];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = threadIdx.x + i * kQThreads;
    if (c < nch) {
      cache[i] = row[c];
      float x[8];
      unpack8(cache[i], x);
      amax = fmaxf(amax, absmax8(x));
    }
  }
  for (int c = threadIdx.x + 4 * kQThreads; c < nch; c += kQThreads) {
    float x[8];
    unpack8(row[c], x);
    amax = fmaxf(amax, absmax8(x));
  }
  amax = block_max(amax, red);
  const float s = scale_of_amax<INT8>(amax);
  if (threadIdx.x == 0) scale[r] = s;
  uint2* qrow = reinterpret_cast<uint2*>(q + (size_t)r * K);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = threadIdx.x + i * kQThreads;
    if (c < nch) {
      float x[8];
      unpack8(cache[i], x);
      qrow[c] = quant8<INT8>(x, s);
    }
  }
  for (int c = threadIdx.x + 4 * kQThreads; c < nch; c += kQThreads) {
    float x[8];
    unpack8(row[c], x);
    qrow[c] = quant8<INT8>(x, s);
  }
}

// ------------------------------------------- Block_FP8 activation groups --
// 16 threads per 1x128 group, 8 elements each.
__global__ void __launch_bounds__(kQThreads) quant_act_groups_kernel(
    const __nv_bfloat16* __restrict__ X, int M, int K, int ldx, uint8_t* __restrict__ q,
    float* __restrict__ scale) {
  // let the next kernel (the GEMM) start streaming its weights now; it
  // waits for this kernel's completion before it reads what we write
  griddep_launch_dependents();
  griddep_wait();
  const int G = K / 128;
  const long long gid = (long long)blockIdx.x * (kQThreads / 16) + (threadIdx.x >> 4);
  const int sub = threadIdx.x & 15;
  const bool valid = gid < (long long)M * G;
  const int m = valid ? (int)(gid / G) : 0;
  const int g = valid ? (int)(gid % G) : 0;
  float x[8];
  if (valid) {
    const uint4 v = reinterpret_cast<const uint4*>(X + (size_t)m * ldx + g * 128)[sub];
    unpack8(v, x);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = 0.f;
  }
  float amax = absmax8(x);
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = scale_of_amax<false>(amax);
  if (valid) {
    if (sub == 0) scale[(size_t)m * G + g] = s;
    reinterpret_cast<uint2*>(q + (size_t)m * K + g * 128)[sub] = quant8<false>(x, s);
  }
}

// --------------------------------------------- Block_FP8 weight blocks --
// One CTA per 128x128 block: 256 threads x 8 chunks of 8 elements.
__global__ void __launch_bounds__(kQThreads) quant_weight_blocks_kernel(
    const __nv_bfloat16* __restrict__ W, int N, int K, uint8_t* __restrict__ q,
    float* __restrict__ scale) {
  __shared__ float red[32];
  // let the next kernel (the GEMM) start streaming its weights now; it
  // waits for this kernel's completion before it reads what we write
  griddep_launch_dependents();
  griddep_wait();
  const int G = K / 128;
  const int nb = blockIdx.x / G, g = blockIdx.x % G;
  float x[8][8];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int idx = threadIdx.x + i * kQThreads;  // 0..2047
    const int r = idx >> 4, c = idx & 15;
    const int n = nb * 128 + r;
    if (n < N) {
      unpack8(reinterpret_cast<const uint4*>(W + (size_t)n * K + g * 128)[c], x[i]);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) x[i][j] = 0.f;
    }
    amax = fmaxf(amax, absmax8(x[i]));
  }
  amax = block_max(amax, red);
  const float s = scale_of_amax<false>(amax);
  if (threadIdx.x == 0) scale[(size_t)nb * G + g] = s;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int idx = threadIdx.x + i * kQThreads;
    const int r = idx >> 4, c = idx & 15;
    const int n = nb * 128 + r;
    if (n < N) reinterpret_cast<uint2*>(q + (size_t)n * K + g * 128)[c] = quant8<false>(x[i], s);
  }
}

// --------------------------------------------------------------- NVFP4 --
// Phase 1: per-CTA partial amax of the tensor (grid-stride, 16-byte loads).
__global__ void __launch_bounds__(kQThreads) nvfp4_amax_kernel(const __nv_bfloat16* __restrict__ X,
                                                               int R, int K, int ldx,
                                                               float* __restrict__ partial) {
  __shared__ float red[32];
  griddep_launch_dependents();
  griddep_wait();
  const int nch = K / 8;
  const long long total = (long long)R * nch;
  float amax = 0.f;
  for (long long i = blockIdx.x * (long long)kQThreads + threadIdx.x; i < total;
       i += (long long)gridDim.x * kQThreads) {
    const int r = (int)(i / nch), c = (int)(i % nch);
    float x[8];
    unpack8(reinterpret_cast<const uint4*>(X + (size_t)r * ldx)[c], x);
    amax = fmaxf(amax, absmax8(x));
  }
  amax = block_max(amax, red);
  if (threadIdx.x == 0) partial[blockIdx.x] = amax;
}

// Inclusive prefix sum over the block's threads (kQThreads of them).
__device__ int block_incl_scan(int v, int* warp_tot) {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, v, d);
    if (l >= d) v += t;
  }
  if (l == 31) warp_tot[w] = v;
  __syncthreads();
  for (int j = 0; j < w; ++j) v += warp_tot[j];
  return v;
}

// Phase 2: one thread per 16-element block (s, c) of the padded scale
// matrix [R_pad, C]; writes 8 bytes of codes and one scale byte (0 in the
// padding).  Every CTA reduces the phase-1 partials itself (deterministic).
// Grouped layout (offsets != NULL): tokens sorted by expert, and expert e's
// scale rows start at 128 x (the 128-row atoms of the experts before it), so
// each expert's first token opens a fresh atom; scale row s holds token
// offsets[e] + (s - first row of e) of the expert e whose rows contain s, or
// padding.  Offsets are clamped to [0, R] as the grouped GEMM does.
__global__ void __launch_bounds__(kQThreads) nvfp4_quant_kernel(
    const __nv_bfloat16* __restrict__ X, int R, int K, int ldx, const float* __restrict__ partial,
    int npartial, const float* __restrict__ static_amax, uint8_t* __restrict__ q,
    uint8_t* __restrict__ sf, float* __restrict__ gscale, int R_pad, int C,
    const int* __restrict__ offsets, int experts) {
  __shared__ float red[32];
  __shared__ int e_tok[kQThreads];             // grouped: expert's first token
  __shared__ int e_cnt[kQThreads];             //          its tokens
  __shared__ int e_row[kQThreads];             //          its first scale row
  __shared__ int warp_tot[kQThreads / 32];
  // let the next kernel (the GEMM) start streaming its weights now; it
  // waits for this kernel's completion before it reads what we write
  griddep_launch_dependents();
  griddep_wait();
  float amax_t = 0.f;
  if (static_amax != nullptr) {
    amax_t = __ldg(static_amax);
  } else {
    for (int i = threadIdx.x; i < npartial; i += kQThreads) amax_t = fmaxf(amax_t, partial[i]);
    amax_t = block_max(amax_t, red);
  }
  const float g = amax_t > 0.f ? __fdiv_rn(amax_t, 2688.f) : 1.f;
  if (blockIdx.x == 0 && threadIdx.x == 0) *gscale = g;
  if (offsets != nullptr) {
    const int t = threadIdx.x;
    int lo = 0, cnt = 0;
    if (t < experts) {
      lo = min(max(__ldg(offsets + t), 0), R);
      cnt = max(min(max(__ldg(offsets + t + 1), 0), R) - lo, 0);
    }
    const int atoms = (cnt + 127) / 128;
    const int incl = block_incl_scan(atoms, warp_tot);
    e_tok[t] = lo;
    e_cnt[t] = cnt;
    e_row[t] = (incl - atoms) * 128;
    __syncthreads();
  }
  const int KS = K / 16;
  const long long total = (long long)R_pad * C;
  for (long long i = blockIdx.x * (long long)kQThreads + threadIdx.x; i < total;
       i += (long long)gridDim.x * kQThreads) {
    const int srow = (int)(i / C), c = (int)(i % C);
    int r = srow;                              // token whose scales sit in row srow
    if (offsets != nullptr) {
      // the last expert whose first scale row is <= srow (an empty expert
      // shares its first row with the next one, which wins)
      int lo = 0, hi = experts - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (e_row[mid] <= srow) lo = mid;
        else hi = mid - 1;
      }
      const int j = srow - e_row[lo];
      r = j < e_cnt[lo] ? e_tok[lo] + j : R;
    }
    uint32_t code = 0;
    if (r < R && c < KS) {
      const uint4* src = reinterpret_cast<const uint4*>(X + (size_t)r * ldx + c * 16);
      float x0[8], x1[8];
      unpack8(src[0], x0);
      unpack8(src[1], x1);
      const float amax_b = fmaxf(absmax8(x0), absmax8(x1));
      const float t = __fdiv_rn(__fdiv_rn(amax_b, 6.f), g);
      code = cvt_e4m3x2(t, 0.f) & 0xFF;
      const float d = __fmul_rn(dec_e4m3(code), g);
      uint2 packed = make_uint2(0u, 0u);
      if (d != 0.f) {
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = __fdiv_rn(x0[j], d);
        packed.x = cvt_e2m1x8(v);
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = __fdiv_rn(x1[j], d);
        packed.y = cvt_e2m1x8(v);
      }
      reinterpret_cast<uint2*>(q + (size_t)r * (K / 2) + c * 8)[0] = packed;
    }
    // 128x4 tiled scale layout
    const size_t atom = (size_t)(srow / 128) * (C / 4) + (c / 4);
    sf[atom * 512 + (srow % 32) * 16 + ((srow % 128) / 32) * 4 + (c % 4)] = (uint8_t)code;
  }
}

}  // namespace

// ------------------------------------------------------------ launchers --
static cudaError_t launch(const void* fn, dim3 grid, dim3 block, void** args, cudaStream_t st,
                          bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelExC(&cfg, fn, args);
}

cudaError_t launch_quant_rows(bool int8, const void* X, int R, int K, int ldx, void* q,
                              float* scale, cudaStream_t st, bool pdl) {
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(X);
  uint8_t* qq = static_cast<uint8_t*>(q);
  void* args[] = {(void*)&x, (void*)&K, (void*)&ldx, (void*)&qq, (void*)&scale};
  const void* fn = int8 ? (const void*)quant_rows_kernel<true> : (const void*)quant_rows_kernel<false>;
  return launch(fn, dim3(R), dim3(kQThreads), args, st, pdl);
}

cudaError_t launch_quant_act_groups(const void* X, int M, int K, int ldx, void* q, float* scale,
                                    cudaStream_t st, bool pdl) {
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(X);
  uint8_t* qq = static_cast<uint8_t*>(q);
  const long long groups = (long long)M * (K / 128);
  const int per_cta = kQThreads / 16;
  dim3 grid((unsigned)((groups + per_cta - 1) / per_cta));
  void* args[] = {(void*)&x, (void*)&M, (void*)&K, (void*)&ldx, (void*)&qq, (void*)&scale};
  return launch((const void*)quant_act_groups_kernel, grid, dim3(kQThreads), args, st, pdl);
}

cudaError_t launch_quant_weight_blocks(const void* W, int N, int K, void* q, float* scale,
                                       cudaStream_t st, bool pdl) {
  const __nv_bfloat16* w = static_cast<const __nv_bfloat16*>(W);
  uint8_t* qq = static_cast<uint8_t*>(q);
  dim3 grid((unsigned)(((N + 127) / 128) * (K / 128)));
  void* args[] = {(void*)&w, (void*)&N, (void*)&K, (void*)&qq, (void*)&scale};
  return launch((const void*)quant_weight_blocks_kernel, grid, dim3(kQThreads), args, st, pdl);
}

int nvfp4_amax_ctas(int R, int K) {
  const long long chunks = (long long)R * (K / 8);
  long long ctas = (chunks + kQThreads - 1) / kQThreads;
  if (ctas > kNvfp4AmaxMaxCtas) ctas = kNvfp4AmaxMaxCtas;
  return (int)(ctas < 1 ? 1 : ctas);
}

cudaError_t launch_quant_nvfp4(const void* X, int R, int K, int ldx, const float* static_amax,
                               void* q, void* sf, float* gscale, float* partial,
                               cudaStream_t st, bool pdl, const int* offsets, int experts) {
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(X);
  int npartial = 0;
  cudaError_t e = cudaSuccess;
  if (static_amax == nullptr) {
    npartial = nvfp4_amax_ctas(R, K);
    void* a1[] = {(void*)&x, (void*)&R, (void*)&K, (void*)&ldx, (void*)&partial};
    e = launch((const void*)nvfp4_amax_kernel, dim3(npartial), dim3(kQThreads), a1, st, pdl);
    if (e != cudaSuccess) return e;
  }
  // scale rows: whole 128-row atoms; grouped, every active expert (at most
  // a = min(experts, R)) may open a fresh atom: floor((R - a) / 128) + a atoms
  int R_pad = ((R + 127) / 128) * 128;
  if (offsets != nullptr) {
    const int a = experts < R ? experts : R;
    R_pad = ((R - a) / 128 + a) * 128;
  }
  int C = ((K + 255) / 256) * 16;
  uint8_t* qq = static_cast<uint8_t*>(q);
  uint8_t* sff = static_cast<uint8_t*>(sf);
  const long long total = (long long)R_pad * C;
  long long ctas = (total + kQThreads - 1) / kQThreads;
  if (ctas > 148 * 16) ctas = 148 * 16;
  const float* pp = partial;
  void* a2[] = {(void*)&x,   (void*)&R,           (void*)&K,  (void*)&ldx,   (void*)&pp,
                (void*)&npartial, (void*)&static_amax, (void*)&qq, (void*)&sff, (void*)&gscale,
                (void*)&R_pad, (void*)&C, (void*)&offsets, (void*)&experts};
  return launch((const void*)nvfp4_quant_kernel, dim3((unsigned)ctas), dim3(kQThreads), a2, st, pdl);
}

}  // namespace qg
