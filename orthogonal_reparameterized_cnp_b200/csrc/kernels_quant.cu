// Int8 base weight (POET-X technical summary section 2.6, POET-XQ: training on a low-bit
// base model whose weight is dequantised on the fly when it is needed).
//
// Per-row symmetric quantisation: s_i = max_j |w_ij| / 127, q_ij = round-to-nearest-even
// (w_ij / s_i) clamped to [-127, 127]; an all-zero row has s_i = 0 and q = 0.  Both the
// scale and the code are decided in fp32 with IEEE division (__fdiv_rn), so the codes are
// reproducible bit for bit.  Dequantisation writes bf16(s_i * q_ij) (fp32 product,
// round to nearest even) for the tcgen05 GEMMs.
#include <cuda_bf16.h>

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

// out[i, j] = bf16(s_i * q_ij); 16 codes per thread when n % 16 == 0 (16-byte accesses)
__global__ void k_dequant_rows_v16(const int8_t* __restrict__ q, const float* __restrict__ s,
                                   __nv_bfloat16* __restrict__ out, int m, int n) {
  const int64_t nv = (int64_t)m * (n / 16);
  for (int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; v < nv;
       v += (int64_t)gridDim.x * blockDim.x) {
    const int64_t e0 = v * 16;
    const int i = (int)(e0 / n);
    const float sc = __ldg(s + i);
    const int4 c = __ldg(reinterpret_cast<const int4*>(q + e0));
    const int w[4] = {c.x, c.y, c.z, c.w};
    uint32_t o[8];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float lo = sc * (float)(int8_t)((w[t] >> (16 * h)) & 0xff);
        const float hi = sc * (float)(int8_t)((w[t] >> (16 * h + 8)) & 0xff);
        const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
        o[t * 2 + h] = *reinterpret_cast<const uint32_t*>(&p);
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(out + e0);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
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

cudaError_t launch_dequant_rows(const int8_t* q, const float* s, void* out, int m, int n,
                                cudaStream_t st) {
  if (m <= 0 || n <= 0) return cudaSuccess;
  const int grid = num_sms() * 8;
  begin_launch("quant", st);
  if (n % 16 == 0 && (reinterpret_cast<uintptr_t>(q) & 15) == 0 &&
      (reinterpret_cast<uintptr_t>(out) & 15) == 0)
    k_dequant_rows_v16<<<grid, 256, 0, st>>>(q, s, static_cast<__nv_bfloat16*>(out), m, n);
  else
    k_dequant_rows<<<grid, 256, 0, st>>>(q, s, static_cast<__nv_bfloat16*>(out), m, n);
  end_launch("quant", st);
  return cudaGetLastError();
}

}  // namespace poetx
