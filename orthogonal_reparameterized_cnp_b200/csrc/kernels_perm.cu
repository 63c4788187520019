// Index-map permutation kernels (POET-X technical summary, section 2.2: permutations are
// applied by remapping indices, never as permutation matrices).
//
// out[r, c] = in[row_idx ? row_idx[r] : r, col_idx[c]]
//
// The permutation acts along the contiguous feature axis of a row-major matrix, so a
// direct gather from global memory would touch a 32-byte sector per element.  Instead
// source rows are staged in shared memory with coalesced 16-byte loads and the permuted
// rows written with coalesced 16-byte stores; the random access happens only in shared
// memory.  HBM traffic is exactly one read and one write of the matrix.  For 2-byte
// elements (the bf16 layer) k_gather_il8 interleaves 8 rows per shared-memory word so
// that one access serves a column of 8 rows (rows narrower than 2048); the row-staged
// kernels cover fp32 and wider rows.
#include <cuda_bf16.h>

#include "poetx_internal.h"

namespace poetx {
namespace {

constexpr int kGatherThreads = 128;
constexpr int kMaxSmemRowBytes = 200 * 1024;

__device__ __forceinline__ uint4 ldg_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

template <typename E>
__global__ void __launch_bounds__(kGatherThreads)
    k_gather_rows_smem(const E* __restrict__ in, E* __restrict__ out,
                       const int32_t* __restrict__ row_idx, const int32_t* __restrict__ col_idx,
                       int rows, int cols, int64_t ld_in, int64_t ld_out) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  E* srow = reinterpret_cast<E*>(smem_raw);
  constexpr int V = 16 / sizeof(E);  // elements per 16-byte vector
  const unsigned ucols = (unsigned)cols;
  for (int r = blockIdx.x; r < rows; r += gridDim.x) {
    int sr = row_idx ? row_idx[r] : r;
    sr = min(max(sr, 0), rows - 1);  // keep the read inside the matrix
    const E* src = in + (int64_t)sr * ld_in;
    const bool vin = (cols % V == 0) && ((reinterpret_cast<uintptr_t>(src) & 15) == 0);
    if (vin) {
      const uint4* s4 = reinterpret_cast<const uint4*>(src);
      uint4* d4 = reinterpret_cast<uint4*>(srow);
      for (int i = threadIdx.x; i < cols / V; i += blockDim.x) d4[i] = ldg_stream(s4 + i);
    } else {
      for (int i = threadIdx.x; i < cols; i += blockDim.x) srow[i] = src[i];
    }
    __syncthreads();
    E* dst = out + (int64_t)r * ld_out;
    const bool vout = (cols % V == 0) && ((reinterpret_cast<uintptr_t>(dst) & 15) == 0);
    if (vout) {
      for (int c0 = threadIdx.x * V; c0 < cols; c0 += blockDim.x * V) {
        E v[V];
#pragma unroll
        for (int e = 0; e < V; ++e) {
          unsigned ci = (unsigned)__ldg(col_idx + c0 + e);
          v[e] = srow[ci < ucols ? ci : ucols - 1];
        }
        *reinterpret_cast<uint4*>(dst + c0) = *reinterpret_cast<const uint4*>(v);
      }
    } else {
      for (int c = threadIdx.x; c < cols; c += blockDim.x) {
        unsigned ci = (unsigned)__ldg(col_idx + c);
        dst[c] = srow[ci < ucols ? ci : ucols - 1];
      }
    }
    __syncthreads();
  }
}

// Pipelined variant for rows whose byte size is a multiple of 16: batches of R rows are
// copied into shared memory with cp.async (two buffers: the next batch lands while the
// current one is gathered), and each thread keeps the index map of the output vectors it
// owns in registers for the CTA's whole life.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait1() {
  asm volatile("cp.async.wait_group 1;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

constexpr int kPipeThreads = 256;

template <typename E, int MAXV>
__global__ void __launch_bounds__(kPipeThreads)
    k_gather_rows_pipe(const E* __restrict__ in, E* __restrict__ out,
                       const int32_t* __restrict__ row_idx, const int32_t* __restrict__ col_idx,
                       int rows, int cols, int64_t ld_in, int64_t ld_out, int R) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  constexpr int V = 16 / sizeof(E);
  const int nvec = cols / V;                    // 16-byte vectors per row
  const int row_elems = cols;                   // elements per staged row
  E* buf[2] = {reinterpret_cast<E*>(smem_raw),
               reinterpret_cast<E*>(smem_raw) + (size_t)R * row_elems};
  const unsigned ucols = (unsigned)cols;

  // index map of the output vectors this thread owns (v = tid + j * blockDim.x), two
  // 16-bit column indices per register (cols <= 65535 on this path)
  uint32_t idx[MAXV][V / 2];
  int myv = 0;
#pragma unroll
  for (int j = 0; j < MAXV; ++j) {
    const int v = threadIdx.x + j * kPipeThreads;
    if (v < nvec) {
      ++myv;
#pragma unroll
      for (int e = 0; e < V; e += 2) {
        unsigned c0 = (unsigned)__ldg(col_idx + v * V + e);
        unsigned c1 = (unsigned)__ldg(col_idx + v * V + e + 1);
        c0 = c0 < ucols ? c0 : ucols - 1;
        c1 = c1 < ucols ? c1 : ucols - 1;
        idx[j][e / 2] = c0 | (c1 << 16);
      }
    }
  }

  const int nbatch = (rows + R - 1) / R;
  // the thread's first (row, vector) of a batch and the step between its copies, so that
  // the copy loop needs no division
  const int rr_first = threadIdx.x / nvec, vv_first = threadIdx.x - rr_first * nvec;
  const int rr_step = kPipeThreads / nvec, vv_step = kPipeThreads - rr_step * nvec;
  auto issue = [&](int batch, E* dst) {
    const int r0 = batch * R;
    const int nr = min(R, rows - r0);
    for (int rr = rr_first, vv = vv_first; rr < nr;) {
      int sr = row_idx ? row_idx[r0 + rr] : r0 + rr;
      sr = min(max(sr, 0), rows - 1);
      cp_async16(dst + (size_t)rr * row_elems + vv * V, in + (int64_t)sr * ld_in + vv * V);
      rr += rr_step;
      vv += vv_step;
      if (vv >= nvec) {
        vv -= nvec;
        ++rr;
      }
    }
  };

  int batch = blockIdx.x;
  int it = 0;
  if (batch < nbatch) issue(batch, buf[0]);
  cp_async_commit();
  for (; batch < nbatch; batch += gridDim.x, ++it) {
    const int next = batch + gridDim.x;
    if (next < nbatch) issue(next, buf[(it + 1) & 1]);
    cp_async_commit();
    cp_async_wait1();
    __syncthreads();
    const E* src = buf[it & 1];
    const int r0 = batch * R;
    const int nr = min(R, rows - r0);
    for (int rr = 0; rr < nr; ++rr) {
      const E* srow = src + (size_t)rr * row_elems;
      E* drow = out + (int64_t)(r0 + rr) * ld_out;
#pragma unroll
      for (int j = 0; j < MAXV; ++j) {
        if (j < myv) {
          E v[V];
#pragma unroll
          for (int e = 0; e < V; e += 2) {
            v[e] = srow[idx[j][e / 2] & 0xFFFFu];
            v[e + 1] = srow[idx[j][e / 2] >> 16];
          }
          *reinterpret_cast<uint4*>(drow + (threadIdx.x + j * kPipeThreads) * V) =
              *reinterpret_cast<const uint4*>(v);
        }
      }
    }
    __syncthreads();
  }
}

// 8-row interleaved variant for 2-byte elements.  Groups of 8 source rows stream into a
// two-deep ring of row-major stages with cp.async.  Each thread then takes an 8 x 8 block
// (8 rows x one 16-byte column chunk) of the current stage, transposes it in registers
// and stores one 16-byte word per column holding that column for all 8 rows.  The
// permutation reads one such word per output column (8 rows at a time, instead of a
// 2-byte word per row and column), transposes back in registers and writes 8 coalesced
// 16-byte row segments.  The word of column c sits at slot c ^ ((c >> 3) & 7), so the 8
// lanes of a store phase, which hold columns 8l + u, hit 8 different bank groups.
constexpr int kIlThreads = 256;
constexpr size_t kIlMaxSmem = 200 * 1024;
// shared memory of the variant with NS stages (NS row groups of 16 bytes a column, plus the
// interleaved words)
constexpr size_t il_smem(int ns, int cols) { return (size_t)(ns * 16 + 16) * cols; }

__device__ __forceinline__ int il_slot(int c) { return c ^ ((c >> 3) & 7); }
__device__ __forceinline__ uint32_t u4_word(const uint4& v, int w) {
  return w == 0 ? v.x : w == 1 ? v.y : w == 2 ? v.z : v.w;
}

template <int MAXC, int NS>
__global__ void __launch_bounds__(kIlThreads, 1)
    k_gather_il8(const uint16_t* __restrict__ in, uint16_t* __restrict__ out,
                 const int32_t* __restrict__ row_idx, const int32_t* __restrict__ col_idx,
                 int rows, int cols, int64_t ld_in, int64_t ld_out) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  // [NS stages of 8 rows x cols] [interleaved words: cols x 16 bytes]
  uint16_t* const stage0 = reinterpret_cast<uint16_t*>(smem_raw);
  uint4* const il = reinterpret_cast<uint4*>(smem_raw + (size_t)NS * 8 * cols * 2);
  const int nchunk = cols / 8;
  pdl_trigger();
  pdl_wait();
  const unsigned ucols = (unsigned)cols;
  // slots of the source columns of the output chunks this thread owns (2 x 16 bit a word)
  uint32_t src[MAXC][4];
#pragma unroll
  for (int j = 0; j < MAXC; ++j) {
    const int q = threadIdx.x + j * kIlThreads;
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      uint32_t v = 0;
      if (q < nchunk) {
        unsigned c0 = (unsigned)__ldg(col_idx + 8 * q + e);
        unsigned c1 = (unsigned)__ldg(col_idx + 8 * q + e + 1);
        c0 = c0 < ucols ? c0 : ucols - 1;
        c1 = c1 < ucols ? c1 : ucols - 1;
        v = (uint32_t)il_slot((int)c0) | ((uint32_t)il_slot((int)c1) << 16);
      }
      src[j][e / 2] = v;
    }
  }
  const int ngroups = (rows + 7) / 8;
  // rows of group g into stage st (rows past the end are not fetched; their words are
  // never written out)
  auto issue = [&](int g, int st) {
    if (g < ngroups) {
      uint16_t* dst = stage0 + (size_t)st * 8 * cols;
      for (int i = threadIdx.x; i < 8 * nchunk; i += kIlThreads) {
        const int r = i / nchunk, q = i - r * nchunk;
        const int row = g * 8 + r;
        if (row < rows) {
          int sr = row_idx ? row_idx[row] : row;
          sr = min(max(sr, 0), rows - 1);
          cp_async16(dst + (size_t)r * cols + 8 * q, in + (int64_t)sr * ld_in + 8 * q);
        }
      }
    }
    cp_async_commit();
  };
  const int step = gridDim.x;
  int g = blockIdx.x;
  if (g >= ngroups) return;
#pragma unroll
  for (int st = 0; st < NS - 1; ++st) issue(g + st * step, st);
  for (int it = 0; g < ngroups; g += step, ++it) {
    const int st = it % NS;
    issue(g + (NS - 1) * step, (it + NS - 1) % NS);
    cp_async_wait<NS - 1>();
    __syncthreads();  // stage st complete; every thread is done reading il
    const uint16_t* sg = stage0 + (size_t)st * 8 * cols;
#pragma unroll
    for (int j = 0; j < MAXC; ++j) {  // stage -> interleaved words
      const int q = threadIdx.x + j * kIlThreads;
      if (q >= nchunk) continue;
      uint4 ld[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) ld[r] = *reinterpret_cast<const uint4*>(sg + (size_t)r * cols + 8 * q);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int w = c >> 1;
        const uint32_t sel = (c & 1) ? 0x7632u : 0x5410u;
        uint4 v;
        v.x = __byte_perm(u4_word(ld[0], w), u4_word(ld[1], w), sel);
        v.y = __byte_perm(u4_word(ld[2], w), u4_word(ld[3], w), sel);
        v.z = __byte_perm(u4_word(ld[4], w), u4_word(ld[5], w), sel);
        v.w = __byte_perm(u4_word(ld[6], w), u4_word(ld[7], w), sel);
        il[il_slot(8 * q + c)] = v;
      }
    }
    __syncthreads();  // words complete; stage st may be refilled
#pragma unroll
    for (int j = 0; j < MAXC; ++j) {  // interleaved words -> 8 permuted row segments
      const int q = threadIdx.x + j * kIlThreads;
      if (q >= nchunk) continue;
      uint4 col[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) col[e] = il[(src[j][e >> 1] >> (16 * (e & 1))) & 0xFFFFu];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int row = g * 8 + r;
        if (row >= rows) break;
        const int w = r >> 1;
        const uint32_t sel = (r & 1) ? 0x7632u : 0x5410u;
        uint4 o;
        o.x = __byte_perm(u4_word(col[0], w), u4_word(col[1], w), sel);
        o.y = __byte_perm(u4_word(col[2], w), u4_word(col[3], w), sel);
        o.z = __byte_perm(u4_word(col[4], w), u4_word(col[5], w), sel);
        o.w = __byte_perm(u4_word(col[6], w), u4_word(col[7], w), sel);
        *reinterpret_cast<uint4*>(out + (int64_t)row * ld_out + 8 * q) = o;
      }
    }
  }
  cp_async_wait<0>();
}

template <int MAXC, int NS>
cudaError_t il8_launch(const void* in, void* out, const int32_t* row_idx, const int32_t* col_idx,
                       int rows, int cols, int64_t ld_in, int64_t ld_out, cudaStream_t s) {
  const size_t smem = il_smem(NS, cols);
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k_gather_il8<MAXC, NS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kIlMaxSmem);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  const int ngroups = (rows + 7) / 8;
  int per_sm = (int)((220 * 1024) / (smem + 1024));
  per_sm = per_sm < 1 ? 1 : (per_sm > 2 ? 2 : per_sm);
  int grid = num_sms() * per_sm;
  if (grid > ngroups) grid = ngroups;
  begin_launch("permute", s);
  const cudaError_t e = launch_pdl(k_gather_il8<MAXC, NS>, dim3(grid), dim3(kIlThreads), smem, s,
                                   static_cast<const uint16_t*>(in), static_cast<uint16_t*>(out),
                                   row_idx, col_idx, rows, cols, ld_in, ld_out);
  end_launch("permute", s);
  return e;
}

// Rows too wide for shared memory: gather straight from global memory (L2 absorbs the
// sector waste; only used beyond ~100k bf16 columns).
template <typename E>
__global__ void __launch_bounds__(256)
    k_gather_rows_direct(const E* __restrict__ in, E* __restrict__ out,
                         const int32_t* __restrict__ row_idx,
                         const int32_t* __restrict__ col_idx, int rows, int cols, int64_t ld_in,
                         int64_t ld_out) {
  const unsigned ucols = (unsigned)cols;
  for (int r = blockIdx.x; r < rows; r += gridDim.x) {
    int sr = row_idx ? row_idx[r] : r;
    sr = min(max(sr, 0), rows - 1);
    const E* src = in + (int64_t)sr * ld_in;
    E* dst = out + (int64_t)r * ld_out;
    for (int c = threadIdx.x; c < cols; c += blockDim.x) {
      unsigned ci = (unsigned)__ldg(col_idx + c);
      dst[c] = src[ci < ucols ? ci : ucols - 1];
    }
  }
}

template <typename E, int MAXV>
cudaError_t pipe_launch(const void* in, void* out, const int32_t* row_idx, const int32_t* col_idx,
                        int rows, int cols, int64_t ld_in, int64_t ld_out, cudaStream_t s) {
  const size_t row_bytes = (size_t)cols * sizeof(E);
  // R rows per batch: ~32 KB per buffer, two buffers per CTA
  int R = (int)((32 * 1024) / row_bytes);
  R = R < 1 ? 1 : (R > 16 ? 16 : R);
  const size_t smem = 2 * (size_t)R * row_bytes;
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k_gather_rows_pipe<E, MAXV>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  const int nbatch = (rows + R - 1) / R;
  int per_sm = (int)((200 * 1024) / (smem + 1024));
  per_sm = per_sm < 1 ? 1 : (per_sm > 8 ? 8 : per_sm);
  int grid = num_sms() * per_sm;
  if (grid > nbatch) grid = nbatch;
  begin_launch("permute", s);
  k_gather_rows_pipe<E, MAXV><<<grid, kPipeThreads, smem, s>>>(
      static_cast<const E*>(in), static_cast<E*>(out), row_idx, col_idx, rows, cols, ld_in,
      ld_out, R);
  end_launch("permute", s);
  return cudaGetLastError();
}

template <typename E>
cudaError_t gather_impl(const void* in, void* out, const int32_t* row_idx,
                        const int32_t* col_idx, int rows, int cols, int64_t ld_in,
                        int64_t ld_out, cudaStream_t s) {
  if (rows <= 0 || cols <= 0) return cudaSuccess;
  const size_t row_bytes = ((size_t)cols * sizeof(E) + 15) & ~size_t(15);
  const int sms = num_sms();
  constexpr int V = 16 / sizeof(E);
  const bool vec_ok = (cols % V == 0) && (ld_in % V == 0) && (ld_out % V == 0) &&
                      ((reinterpret_cast<uintptr_t>(in) & 15) == 0) &&
                      ((reinterpret_cast<uintptr_t>(out) & 15) == 0);
  const int nvec = cols / V;
  // interleaved gather (4-deep stage ring) for rows narrower than 2048 bf16, where it
  // measured 1.1-1.2x the row-batched pipeline (256-1024 columns); from 2048 columns on
  // the pipeline is as fast or faster (+5% at 2048, +19% at 2560, +10% at 4096 against the
  // interleaved forms that fit there)
  if (sizeof(E) == 2 && vec_ok && cols < 8 * kIlThreads && il_smem(4, cols) <= kIlMaxSmem)
    return il8_launch<1, 4>(in, out, row_idx, col_idx, rows, cols, ld_in, ld_out, s);
  if (vec_ok && cols <= 65535 && nvec <= 8 * kPipeThreads && 2 * row_bytes <= 96 * 1024) {
    const int need = (nvec + kPipeThreads - 1) / kPipeThreads;
    if (need <= 1) return pipe_launch<E, 1>(in, out, row_idx, col_idx, rows, cols, ld_in, ld_out, s);
    if (need <= 2) return pipe_launch<E, 2>(in, out, row_idx, col_idx, rows, cols, ld_in, ld_out, s);
    if (need <= 4) return pipe_launch<E, 4>(in, out, row_idx, col_idx, rows, cols, ld_in, ld_out, s);
    return pipe_launch<E, 8>(in, out, row_idx, col_idx, rows, cols, ld_in, ld_out, s);
  }
  if (row_bytes <= (size_t)kMaxSmemRowBytes) {
    static bool attr_set = false;  // single-device use; the pipelined path covers the rest
    if (!attr_set) {
      cudaError_t e = cudaFuncSetAttribute(k_gather_rows_smem<E>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           kMaxSmemRowBytes);
      if (e != cudaSuccess) return e;
      attr_set = true;
    }
    int per_sm = (int)(200 * 1024 / row_bytes);
    per_sm = per_sm < 1 ? 1 : (per_sm > 16 ? 16 : per_sm);
    int grid = sms * per_sm;
    if (grid > rows) grid = rows;
    begin_launch("permute", s);
    k_gather_rows_smem<E><<<grid, kGatherThreads, row_bytes, s>>>(
        static_cast<const E*>(in), static_cast<E*>(out), row_idx, col_idx, rows, cols, ld_in,
        ld_out);
    end_launch("permute", s);
  } else {
    int grid = sms * 8;
    if (grid > rows) grid = rows;
    begin_launch("permute", s);
    k_gather_rows_direct<E><<<grid, 256, 0, s>>>(static_cast<const E*>(in), static_cast<E*>(out),
                                                 row_idx, col_idx, rows, cols, ld_in, ld_out);
    end_launch("permute", s);
  }
  return cudaGetLastError();
}

__global__ void k_compose_perm(const int32_t* __restrict__ outer, const int32_t* __restrict__ inner,
                               int32_t* __restrict__ out, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    const int j = min(max(inner[i], 0), n - 1);
    out[i] = outer[j];
  }
}

}  // namespace

cudaError_t launch_compose_perm(const int32_t* outer, const int32_t* inner, int32_t* out, int n,
                                cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  begin_launch("permute", s);
  k_compose_perm<<<(n + 255) / 256, 256, 0, s>>>(outer, inner, out, n);
  end_launch("permute", s);
  return cudaGetLastError();
}

cudaError_t launch_gather(const void* in, void* out, const int32_t* row_idx,
                          const int32_t* col_idx, int rows, int cols, int64_t ld_in,
                          int64_t ld_out, int elem_bytes, cudaStream_t s) {
  if (elem_bytes == 2)
    return gather_impl<uint16_t>(in, out, row_idx, col_idx, rows, cols, ld_in, ld_out, s);
  return gather_impl<uint32_t>(in, out, row_idx, col_idx, rows, cols, ld_in, ld_out, s);
}

}  // namespace poetx
