// Cayley-Neumann forward for callers that cannot hand the library a scratch buffer.
//
// Some callers cannot allocate device memory at the point where they need G: a host
// framework that owns every byte of device memory through its own pool and gives this
// call site no access to it, or a latency-critical loop where a cudaMalloc would
// synchronise the device.  poetx_cnp_fwd_static serves them with scratch that lives in
// a fixed array of this library's own device memory, reserved when the library is
// loaded on a GPU and held until the process exits.
//
// The array's name is only a host-side stand-in in host code: a kernel given it would
// fault, or read host memory where the GPU can reach it.  Its device address is looked
// up once per device with cudaGetSymbolAddress and that address is what the kernels get.
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "poetx_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = 32ull << 20;  // 32 MiB on every GPU using the library

static __device__ __align__(256) unsigned char g_cnp_static_scratch[kStaticScratchBytes];

std::mutex g_mu;
void* g_scratch_dev[64] = {nullptr};

// Device address of the array on the current device (looked up on first use).
int static_scratch(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return poetx::cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return poetx::fail(POETX_ERR_INVALID_ARG, "device index out of range");
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_dev[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_cnp_static_scratch);
    if (e != cudaSuccess) return poetx::cuda_fail(e, "cudaGetSymbolAddress(static CNP scratch)");
    g_scratch_dev[dev] = p;
  }
  *out = g_scratch_dev[dev];
  return POETX_OK;
}

}  // namespace

extern "C" int poetx_cnp_fwd_static(const float* theta, float* G, void* G_bf16, int32_t nblk,
                                    int32_t b, int32_t k, void* stream) {
  if (nblk < 0) return poetx::fail(POETX_ERR_INVALID_ARG, "nblk must be >= 0");
  if (b < 1 || b > 1024 || k < 1 || k > 16)
    return poetx::fail(POETX_ERR_SHAPE, "block size b must be in [1, 1024], k in [1, 16]");
  // One block's forward scratch (its d + 2 matrices and counters, plus the call's fixed
  // part) must fit the fixed array; larger counts run in chunks inside it.
  const size_t one_block = poetx::cnp_fwd_block_bytes(b, k) + poetx::cnp_fixed_bytes();
  if (one_block > kStaticScratchBytes)
    return poetx::fail(POETX_ERR_WORKSPACE,
                       "poetx_cnp_fwd_static: one block of size b=" + std::to_string(b) +
                           ", k=" + std::to_string(k) + " needs " + std::to_string(one_block) +
                           " bytes of scratch, above the fixed " +
                           std::to_string(kStaticScratchBytes) +
                           " bytes; use poetx_cnp_fwd with a caller buffer");
  if (nblk == 0) return POETX_OK;
  void* ws = nullptr;
  int st = static_scratch(&ws);
  if (st != POETX_OK) return st;
  return poetx_cnp_fwd(theta, G, G_bf16, nblk, b, k, ws, kStaticScratchBytes, stream);
}
