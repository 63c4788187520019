// FP32 FMA throughput probe: the peak that bounds the SIMT kernels (the Cayley-Neumann
// products are compute-bound on the FP32 FMA pipe), measured on the device at hand rather
// than derived from nominal unit counts and clocks.
//
// Every thread runs kChains independent multiply-add chains a <- a * x + y, so the pipe
// never waits on a result; x and y arrive at run time, so nothing is folded away, and each
// thread stores its sum so that no chain is dead code.  The chains run in packed pairs
// (fma.rn.f32x2, two fp32 FMAs per instruction), the form the CNP product loops use: on
// B200 it reaches a few percent more than one FMA per instruction, whose issue slots then
// limit the pipe.
#include "poetx_internal.h"

namespace poetx {
namespace {

constexpr int kProbeThreads = 512;
constexpr int kChains = 16;

__global__ void __launch_bounds__(kProbeThreads) k_fma_probe(float* out, int iters, float x, float y) {
  unsigned long long a[kChains / 2], xx, yy;
  asm("mov.b64 %0, {%1, %1};" : "=l"(xx) : "f"(x));
  asm("mov.b64 %0, {%1, %1};" : "=l"(yy) : "f"(y));
#pragma unroll
  for (int i = 0; i < kChains / 2; ++i) {
    const float lo = 1e-3f * (float)threadIdx.x + (float)(2 * i), hi = lo + 1.f;
    asm("mov.b64 %0, {%1, %2};" : "=l"(a[i]) : "f"(lo), "f"(hi));
  }
#pragma unroll 4
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < kChains / 2; ++i)
      asm volatile("fma.rn.f32x2 %0, %0, %1, %2;" : "+l"(a[i]) : "l"(xx), "l"(yy));
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kChains / 2; ++i) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(a[i]));
    s += lo + hi;
  }
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
