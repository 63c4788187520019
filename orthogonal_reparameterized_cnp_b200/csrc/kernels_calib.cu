// FP32 FMA throughput probe: the peak that bounds the SIMT kernels (the Cayley-Neumann
// products are compute-bound on the FP32 FMA pipe), measured on the device at hand rather
// than derived from nominal unit counts and clocks.
//
// Every thread runs kChains independent multiply-add chains a <- a * x + y, so the pipe
// never waits on a result; x and y arrive at run time, so nothing is folded away, and each
// thread stores its sum so that no chain is dead code.
#include "poetx_internal.h"

namespace poetx {
namespace {

constexpr int kProbeThreads = 512;
constexpr int kChains = 16;

__global__ void __launch_bounds__(kProbeThreads) k_fma_probe(float* out, int iters, float x, float y) {
  float a[kChains];
#pragma unroll
  for (int i = 0; i < kChains; ++i) a[i] = 1e-3f * (float)threadIdx.x + (float)i;
#pragma unroll 4
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < kChains; ++i) a[i] = fmaf(a[i], x, y);
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kChains; ++i) s += a[i];
  out[(size_t)blockIdx.x * kProbeThreads + threadIdx.x] = s;
}

}  // namespace
}  // namespace poetx

extern "C" int poetx_fma_probe(float* out, int32_t ctas, int32_t iters, void* stream) {
  if (ctas < 1 || iters < 1) return poetx::fail(POETX_ERR_INVALID_ARG, "ctas and iters must be >= 1");
  if (!out) return poetx::fail(POETX_ERR_INVALID_ARG, "null pointer");
  if ((reinterpret_cast<uintptr_t>(out) & 15) != 0)
    return poetx::fail(POETX_ERR_ALIGN, "out must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  poetx::begin_launch("fma_probe", s);
  poetx::k_fma_probe<<<ctas, poetx::kProbeThreads, 0, s>>>(out, iters, 0.9999999f, 1e-7f);
  poetx::end_launch("fma_probe", s);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return poetx::cuda_fail(e, "fma probe launch");
  return POETX_OK;
}
