// Int8 base weight (POET-X technical summary section 2.6, POET-XQ: training on a low-bit
// base model whose weight is dequantised on the fly when it is needed).
//
// Per-row symmetric quantisation: s_i = max_j |w_ij| / 127, q_ij = round-to-nearest-even
// (w_ij / s_i) clamped to [-127, 127]; an all-zero row has s_i = 0 and q = 0.  Both the
// scale and the code are decided in fp32 with IEEE division (__fdiv_rn), so the codes are
// reproducible bit for bit.  Dequantisation writes bf16(s_i * q_ij) (fp32 product,
// round to nearest even) for the tcgen05 GEMMs.
#include <cuda_bf16.h>

#include "dequant_dev.cuh"
#include "poetx_internal.h"

namespace poetx {
namespace {

constexpr int kQThreads = 256;

template <typename E>
__device__ __forceinline__ float to_f32(E v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

// One CTA per row (grid-stride over rows): max |w| by a block reduction, then the codes.
template <typename E>
__global__ void __launch_bounds__(kQThreads)
    k_quantize_rows(const E* __restrict__ W, int8_t* __restrict__ q, float* __restrict__ s,
                    int m, int n) {
  __shared__ float warp_max[kQThreads / 32];
  __shared__ float row_scale;
  for (int i = blockIdx.x; i < m; i += gridDim.x) {
    const E* w = W + (int64_t)i * n;
    float amax = 0.f;
    for (int j = threadIdx.x; j < n; j += kQThreads) amax = fmaxf(amax, fabsf(to_f32(w[j])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = amax;
    __syncthreads();
    if (threadIdx.x == 0) {
      float a = warp_max[0];
      for (int t = 1; t < kQThreads / 32; ++t) a = fmaxf(a, warp_max[t]);
      const float sc = __fdiv_rn(a, 127.0f);
      row_scale = sc;
      s[i] = sc;
    }
    __syncthreads();
    const float sc = row_scale;
    int8_t* qi = q + (int64_t)i * n;
    for (int j = threadIdx.x; j < n; j += kQThreads) {
      float c = 0.f;
      if (sc > 0.f) c = fminf(fmaxf(rintf(__fdiv_rn(to_f32(w[j]), sc)), -127.f), 127.f);
      qi[j] = (int8_t)(int)c;
    }
    __syncthreads();  // warp_max / row_scale are reused by the next row
  }
}

// The int8 merged weight straight from W0: q[i, j] = code of W0[perm_R[i], perm_P[j]] with
// the scale of its row.  A permutation does not change a row's maximum, so the scale is
// that of source row perm_R[i]; the source row is staged in shared memory (coalesced) and
// gathered from there.  The same fp32 decisions as k_quantize_rows on the merged row.
template <typename E>
__global__ void __launch_bounds__(kQThreads)
    k_merge_quantize(const E* __restrict__ W0, const int32_t* __restrict__ perm_R,
                     const int32_t* __restrict__ perm_P, int8_t* __restrict__ q,
                     float* __restrict__ s, int m, int n) {
  extern __shared__ __align__(16) unsigned char row_raw[];
  E* row = reinterpret_cast<E*>(row_raw);
  __shared__ float warp_max[kQThreads / 32];
  __shared__ float row_scale;
  const unsigned un = (unsigned)n, um = (unsigned)m;
  for (int i = blockIdx.x; i < m; i += gridDim.x) {
    unsigned sr = (unsigned)__ldg(perm_R + i);
    sr = sr < um ? sr : um - 1;  // keep the read inside the matrix
    const E* w = W0 + (int64_t)sr * n;
    float amax = 0.f;
    for (int j = threadIdx.x; j < n; j += kQThreads) {
      const E v = w[j];
      row[j] = v;
      amax = fmaxf(amax, fabsf(to_f32(v)));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = amax;
    __syncthreads();
    if (threadIdx.x == 0) {
      float a = warp_max[0];
      for (int t = 1; t < kQThreads / 32; ++t) a = fmaxf(a, warp_max[t]);
      const float sc = __fdiv_rn(a, 127.0f);
      row_scale = sc;
      s[i] = sc;
    }
    __syncthreads();
    const float sc = row_scale;
    int8_t* qi = q + (int64_t)i * n;
    for (int j = threadIdx.x; j < n; j += kQThreads) {
      unsigned c = (unsigned)__ldg(perm_P + j);
      c = c < un ? c : un - 1;
      float code = 0.f;
      if (sc > 0.f) code = fminf(fmaxf(rintf(__fdiv_rn(to_f32(row[c]), sc)), -127.f), 127.f);
      qi[j] = (int8_t)(int)code;
    }
    __syncthreads();  // the staged row, warp_max and row_scale are reused by the next row
  }
}

// out[i, j] = bf16(s_i * q_ij); 16 codes per thread (16-byte accesses)
__global__ void k_dequant_2d(const int8_t* __restrict__ q, int64_t ldq, const float* __restrict__ s,
                             __nv_bfloat16* __restrict__ out, int64_t ldo, int rows, int cols) {
  pdl_trigger();
  pdl_wait();
  dequant_rows2d(q, ldq, s, out, ldo, rows, cols, blockIdx.x * (int64_t)blockDim.x + threadIdx.x,
                 (int64_t)gridDim.x * blockDim.x);
}

__global__ void k_dequant_rows(const int8_t* __restrict__ q, const float* __restrict__ s,
                               __nv_bfloat16* __restrict__ out, int m, int n) {
  const int64_t ne = (int64_t)m * n;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < ne;
       e += (int64_t)gridDim.x * blockDim.x)
    out[e] = __float2bfloat16_rn(__ldg(s + e / n) * (float)q[e]);
}

}  // namespace

cudaError_t launch_quantize_rows(const void* W, int8_t* q, float* s, int m, int n,
                                 int elem_bytes, cudaStream_t st) {
  if (m <= 0) return cudaSuccess;
  int grid = num_sms() * 8;
  if (grid > m) grid = m;
  begin_launch("quant", st);
  if (elem_bytes == 2)
    k_quantize_rows<__nv_bfloat16><<<grid, kQThreads, 0, st>>>(
        static_cast<const __nv_bfloat16*>(W), q, s, m, n);
  else
    k_quantize_rows<float><<<grid, kQThreads, 0, st>>>(static_cast<const float*>(W), q, s, m, n);
  end_launch("quant", st);
  return cudaGetLastError();
}

cudaError_t launch_merge_quantize(const void* W0, const int32_t* perm_R, const int32_t* perm_P,
                                  int8_t* q, float* s, int m, int n, int elem_bytes,
                                  cudaStream_t st) {
  if (m <= 0 || n <= 0) return cudaSuccess;
  const size_t smem = (size_t)n * elem_bytes;
  if (smem > 200 * 1024) return cudaErrorInvalidValue;
  static bool attr_done[2][64] = {{false}};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  cudaError_t e;
  const int es = elem_bytes == 2 ? 0 : 1;
  if (!attr_done[es][dev]) {
    e = elem_bytes == 2
            ? cudaFuncSetAttribute(k_merge_quantize<__nv_bfloat16>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024)
            : cudaFuncSetAttribute(k_merge_quantize<float>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e != cudaSuccess) return e;
    attr_done[es][dev] = true;
  }
  int grid = num_sms() * 4;
  if (grid > m) grid = m;
  begin_launch("quant", st);
  if (elem_bytes == 2)
    k_merge_quantize<__nv_bfloat16><<<grid, kQThreads, smem, st>>>(
        static_cast<const __nv_bfloat16*>(W0), perm_R, perm_P, q, s, m, n);
  else
    k_merge_quantize<float><<<grid, kQThreads, smem, st>>>(static_cast<const float*>(W0), perm_R,
                                                           perm_P, q, s, m, n);
  end_launch("quant", st);
  return cudaGetLastError();
}

cudaError_t launch_dequant_rows(const int8_t* q, const float* s, void* out, int m, int n,
                                cudaStream_t st) {
  if (m <= 0 || n <= 0) return cudaSuccess;
  if (n % 16 == 0 && (reinterpret_cast<uintptr_t>(q) & 15) == 0 &&
      (reinterpret_cast<uintptr_t>(out) & 15) == 0)
    return launch_dequant_2d(q, n, s, out, n, m, n, st);
  const int grid = num_sms() * 8;
  begin_launch("quant", st);
  k_dequant_rows<<<grid, 256, 0, st>>>(q, s, static_cast<__nv_bfloat16*>(out), m, n);
  end_launch("quant", st);
  return cudaGetLastError();
}

cudaError_t launch_dequant_2d(const int8_t* q, int64_t ldq, const float* s, void* out,
                              int64_t ldo, int rows, int cols, cudaStream_t st) {
  if (rows <= 0 || cols <= 0) return cudaSuccess;
  if (cols % 16 != 0 || ldq % 16 != 0 || ldo % 8 != 0 ||
      (reinterpret_cast<uintptr_t>(q) & 15) != 0 || (reinterpret_cast<uintptr_t>(out) & 15) != 0)
    return cudaErrorInvalidValue;
  int grid = num_sms() * 8;
  const int64_t chunks = (int64_t)rows * (cols / 16);
  if ((int64_t)grid * 256 > chunks) grid = (int)((chunks + 255) / 256);
  begin_launch("quant", st);
  const cudaError_t e = launch_pdl(k_dequant_2d, dim3(grid), dim3(256), 0, st, q, ldq, s,
                                   static_cast<__nv_bfloat16*>(out), ldo, rows, cols);
  end_launch("quant", st);
  return e;
}

}  // namespace poetx
