// Device helper shared by the int8 dequantisation kernel and the side warps of the tensor-core
// GEMM: 16 int8 codes of one row -> 16 bf16 values bf16(s * q) (fp32 product, round to
// nearest even), written as two 16-byte vectors.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace poetx {

__device__ __forceinline__ void dequant16_codes(const int4 c, float sc,
                                                __nv_bfloat16* __restrict__ dst) {
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
  uint4* d = reinterpret_cast<uint4*>(dst);
  d[0] = make_uint4(o[0], o[1], o[2], o[3]);
  d[1] = make_uint4(o[4], o[5], o[6], o[7]);
}
__device__ __forceinline__ void dequant16(const int8_t* __restrict__ src, float sc,
                                          __nv_bfloat16* __restrict__ dst) {
  dequant16_codes(__ldg(reinterpret_cast<const int4*>(src)), sc, dst);
}

// dst[r][c] = bf16(scales[r] * q[r][c]) for r < rows, c < cols (cols % 16 == 0; q, dst rows
// 16-byte aligned), chunks of 16 codes handed out from `first` in steps of `stride`.  Four
// chunks per round: their loads are all issued before the first one is converted.
__device__ __forceinline__ void dequant_rows2d(const int8_t* __restrict__ q, int64_t ldq,
                                               const float* __restrict__ scales,
                                               __nv_bfloat16* __restrict__ dst, int64_t ldd,
                                               int rows, int cols, int64_t first,
                                               int64_t stride) {
  const int cpr = cols / 16;
  const int64_t nchunk = (int64_t)rows * cpr;
  constexpr int kIn = 4;
  for (int64_t v0 = first; v0 < nchunk; v0 += kIn * stride) {
    int4 code[kIn];
    float sc[kIn];
    int64_t out[kIn];
#pragma unroll
    for (int u = 0; u < kIn; ++u) {
      const int64_t v = v0 + u * stride;
      out[u] = -1;
      if (v < nchunk) {
        const int r = (int)(v / cpr);
        const int c = (int)(v - (int64_t)r * cpr) * 16;
        code[u] = __ldg(reinterpret_cast<const int4*>(q + (int64_t)r * ldq + c));
        sc[u] = __ldg(scales + r);
        out[u] = (int64_t)r * ldd + c;
      }
    }
#pragma unroll
    for (int u = 0; u < kIn; ++u)
      if (out[u] >= 0) dequant16_codes(code[u], sc[u], dst + out[u]);
  }
}

}  // namespace poetx
