// tcgen05 (5th-generation tensor core) GEMM for sm_100a, fed by TMA.
//
//   D[M x N] = A[M x K] . B[N x K]^T      (bf16 operands, fp32 accumulation in TMEM)
//
// used for every dense contraction of the POET-X layer (technical summary sections
// 2.1-2.3):
//   * the batched block-diagonal products V_j = U_j G_j^T and dW_j = dZ_j G_j (one batch
//     entry per b x b block; the sparse block-diagonal matrix is never formed),
//   * the merged-weight products W = V W0'^T and dV = dW W0',
//   * the block-gradient contractions dG_j = sum_t g_t^T h_t over tokens, split over the
//     token axis into fixed partial sums.
//
// Structure: one persistent CTA per SM, 320 threads.
//   warp 0      TMA producer (one lane): A/B k-chunks of 64 into a STAGES-deep smem ring
//               (or, for the block-diagonal products, A only with the item's whole B
//               resident)
//   warp 1      TMEM allocator + MMA issuer (one lane): 4 x (M=128, N=BN, K=16) per chunk
//   warps 2..9  epilogue: tcgen05.ld of the fp32 accumulator, convert, stage each 32 x 64
//               piece in a 128-byte-swizzled 4 KB tile, TMA tensor store
//   warps 10-11 (SIDE instantiation only): a side job independent of the GEMM -- the
//               int8 weight's next panel dequantised to bf16 while this one is multiplied
// Two TMEM accumulators (2 x BN columns) let the epilogue of tile t overlap the main loop
// of tile t+1.  The kernel is launched as a programmatic dependent of the previous kernel
// on the stream: set-up (barriers, TMEM, tensor-map prefetch) runs before
// griddepcontrol.wait, global memory only after it.  Operands may be K-major or MN-major (transposed) in global memory; both
// are staged with the 128-byte swizzle the UMMA smem descriptors expect.
//
// Every mbarrier wait is bounded: after the wait limit (Params::wait_ns, 2 s unless the
// library's poetx_set_wait_limit changed it) the waiting role records
// POETX_ERR_TIMEOUT in a device flag and leaves its loop; the CTA then drains its
// outstanding TMA loads and MMAs (again with bounded waits), frees TMEM and returns.
// No cluster multicast is used anywhere.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "dequant_dev.cuh"
#include "poetx_internal.h"
#include "umma_ptx.cuh"

namespace poetx {
namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;  // 64 bf16 = 128 bytes = one swizzle row
constexpr int kThreads = 320;  // 2 control warps + 8 epilogue warps
constexpr int kEpiWarps = 8;

// B_RES: the B operand of a whole item (K <= 256) stays in shared memory while the CTA
// works through consecutive items that share it (the block-diagonal products: one G_j
// for many token tiles); only A streams through the ring.
template <int BN, bool B_RES>
struct Cfg {
  static constexpr int A_BYTES = kBM * kBK * 2;
  static constexpr int B_BYTES = BN * kBK * 2;  // one K chunk of B
  static constexpr int STAGES = B_RES ? (BN == 256 ? 4 : 6) : (BN == 256 ? 4 : 6);
  static constexpr int KCH_RES = 4;             // resident K chunks (K <= 256)
  static constexpr int RING_BYTES = B_RES ? STAGES * A_BYTES : STAGES * (A_BYTES + B_BYTES);
  static constexpr int BRES_BYTES = B_RES ? KCH_RES * B_BYTES : 0;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int EPI_BYTES = 8 * 4096;  // one 4 KB TMA-store staging tile per epilogue warp
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = 1024 + RING_BYTES + BRES_BYTES + EPI_BYTES + BAR_BYTES;
};

struct Params {
  int M, N, K, batch, ksplit, kcps, total_kc;
  int tiles_m, tiles_n, num_items;
  int a_boff_mn, a_boff_k, b_boff_mn, b_boff_k;
  void* D;
  int out_f32;
  long long ldd, d_boff_col, d_boff, d_split;
  int* err;
  unsigned long long wait_ns;  // bound of every mbarrier wait
  int y_per_bz, y_per_split;  // output tensor rows per batch entry / per split
  // side job (SIDE instantiation)
  const int8_t* side_q;
  long long side_ldq, side_ldd;
  const float* side_scales;
  __nv_bfloat16* side_dst;
  int side_rows, side_cols;
};
constexpr int kSideWarps = 2;

template <int BN, bool A_MN, bool B_MN>
__device__ __forceinline__ uint32_t make_idesc() {
  return (1u << 4)                         // D format: f32
         | (1u << 7)                       // A format: bf16
         | (1u << 10)                      // B format: bf16
         | ((A_MN ? 1u : 0u) << 15)        // A major
         | ((B_MN ? 1u : 0u) << 16)        // B major
         | ((uint32_t)(BN >> 3) << 17)     // N
         | ((uint32_t)(kBM >> 4) << 24);   // M
}

struct Item {
  int bz, split, tm, tn;
};
__device__ __forceinline__ Item decode(const Params& p, int item) {
  Item it;
  it.tm = item % p.tiles_m;
  int r = item / p.tiles_m;
  it.tn = r % p.tiles_n;
  r /= p.tiles_n;
  it.split = r % p.ksplit;
  it.bz = r / p.ksplit;
  return it;
}

// Items a CTA works on: round-robin (item = blockIdx.x + q * gridDim.x), or, in B_RES
// mode, one contiguous range so that consecutive items share their B operand.
struct Range {
  int first, last, step;
};
__device__ __forceinline__ Range my_items(const Params& p, bool contiguous) {
  Range r;
  if (contiguous) {
    r.first = (int)(((long long)blockIdx.x * p.num_items) / gridDim.x);
    r.last = (int)(((long long)(blockIdx.x + 1) * p.num_items) / gridDim.x);
    r.step = 1;
  } else {
    r.first = blockIdx.x;
    r.last = p.num_items;
    r.step = gridDim.x;
  }
  return r;
}
__device__ __forceinline__ int b_key(const Params& p, int item) {
  const Item w = decode(p, item);
  return (w.bz * p.ksplit + w.split) * p.tiles_n + w.tn;
}

template <int BN, bool A_MN, bool B_MN, bool B_RES, bool SIDE>
__global__ void __launch_bounds__(kThreads + (SIDE ? 32 * kSideWarps : 0), 1)
    k_umma_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmD, const Params p) {
  using C = Cfg<BN, B_RES>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t sA = base;                                   // STAGES x A_BYTES
  const uint32_t sB = base + C::STAGES * C::A_BYTES;          // ring B (or resident B)
  const uint32_t sEpi = base + C::RING_BYTES + C::BRES_BYTES;  // 1024-aligned staging tiles
  const uint32_t sBar = sEpi + C::EPI_BYTES;
  // barrier block: full[S], empty[S], tfull[2], tempty[2], drain, bfull, bempty, tmem slot
  auto full_bar = [&](int s) { return sBar + 8u * s; };
  auto empty_bar = [&](int s) { return sBar + 8u * (C::STAGES + s); };
  auto tfull_bar = [&](int a) { return sBar + 8u * (2 * C::STAGES + a); };
  auto tempty_bar = [&](int a) { return sBar + 8u * (2 * C::STAGES + 2 + a); };
  const uint32_t drain_bar = sBar + 8u * (2 * C::STAGES + 4);
  const uint32_t bfull_bar = sBar + 8u * (2 * C::STAGES + 5);
  const uint32_t bempty_bar = sBar + 8u * (2 * C::STAGES + 6);
  const uint32_t tmem_slot = sBar + 8u * (2 * C::STAGES + 7);
  unsigned char* generic_base = smem_raw + (base - raw);
  volatile uint32_t* tmem_slot_ptr =
      reinterpret_cast<volatile uint32_t*>(generic_base + (tmem_slot - base));
  // address of B chunk kc for ring stage s (or of resident chunk kc)
  auto b_addr_of = [&](int s, int kc) -> uint32_t {
    return B_RES ? sB + (uint32_t)kc * C::B_BYTES : sB + (uint32_t)s * C::B_BYTES;
  };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Range rng = my_items(p, B_RES);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), kEpiWarps);
    }
    mbar_init(drain_bar, 1);
    mbar_init(bfull_bar, 1);
    mbar_init(bempty_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmD);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot_ptr;
  // set-up done: from here on the previous kernel's results are read
  pdl_trigger();
  pdl_wait();

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    int it = 0;
    int last_round[8];
    for (int s = 0; s < 8; ++s) last_round[s] = -1;
    int brun = -1, cur_key = -1;
    bool ok = true;
    for (int item = rng.first; ok && item < rng.last; item += rng.step) {
      const Item w = decode(p, item);
      const int m0 = w.tm * kBM, n0 = w.tn * BN;
      const int kc0 = w.split * p.kcps;
      const int kc1 = min(p.total_kc, kc0 + p.kcps);
      if (B_RES) {
        const int key = b_key(p, item);
        if (key != cur_key) {
          ++brun;
          if (!mbar_wait(bempty_bar, (brun & 1) ^ 1, p.err, p.wait_ns)) {
            ok = false;
            break;
          }
          mbar_expect_tx(bfull_bar, (uint32_t)(kc1 - kc0) * C::B_BYTES);
          for (int kc = kc0; kc < kc1; ++kc) {
            const int k = kc * kBK;
            const uint32_t b_dst = b_addr_of(0, kc - kc0);
            if (!B_MN) {
              tma_load_2d(b_dst, &tmB, k + w.bz * p.b_boff_k, n0 + w.bz * p.b_boff_mn, bfull_bar);
            } else {
#pragma unroll
              for (int i = 0; i < BN / 64; ++i)
                tma_load_2d(b_dst + i * 8192, &tmB, n0 + 64 * i + w.bz * p.b_boff_mn,
                            k + w.bz * p.b_boff_k, bfull_bar);
            }
          }
          cur_key = key;
        }
      }
      for (int kc = kc0; kc < kc1; ++kc, ++it) {
        const int s = it % C::STAGES, r = it / C::STAGES;
        if (!mbar_wait(empty_bar(s), (r & 1) ^ 1, p.err, p.wait_ns)) {
          ok = false;
          break;
        }
        mbar_expect_tx(full_bar(s), B_RES ? C::A_BYTES : C::A_BYTES + C::B_BYTES);
        last_round[s] = r;
        const int k = kc * kBK;
        const uint32_t a_dst = sA + s * C::A_BYTES;
        if (!A_MN) {
          tma_load_2d(a_dst, &tmA, k + w.bz * p.a_boff_k, m0 + w.bz * p.a_boff_mn, full_bar(s));
        } else {
          tma_load_2d(a_dst, &tmA, m0 + w.bz * p.a_boff_mn, k + w.bz * p.a_boff_k, full_bar(s));
          tma_load_2d(a_dst + 8192, &tmA, m0 + 64 + w.bz * p.a_boff_mn, k + w.bz * p.a_boff_k,
                      full_bar(s));
        }
        if (!B_RES) {
          const uint32_t b_dst = b_addr_of(s, 0);
          if (!B_MN) {
            tma_load_2d(b_dst, &tmB, k + w.bz * p.b_boff_k, n0 + w.bz * p.b_boff_mn, full_bar(s));
          } else {
#pragma unroll
            for (int i = 0; i < BN / 64; ++i)
              tma_load_2d(b_dst + i * 8192, &tmB, n0 + 64 * i + w.bz * p.b_boff_mn,
                          k + w.bz * p.b_boff_k, full_bar(s));
          }
        }
      }
    }
    if (!ok) {
      // make sure no TMA write into this CTA's shared memory is still in flight
      for (int s = 0; s < C::STAGES; ++s)
        if (last_round[s] >= 0) mbar_drain_wait(full_bar(s), last_round[s] & 1);
      if (B_RES && brun >= 0) mbar_drain_wait(bfull_bar, brun & 1);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = make_idesc<BN, A_MN, B_MN>();
    int it = 0, tcount = 0;
    int brun = -1, cur_key = -1;
    bool ok = true;
    for (int item = rng.first; ok && item < rng.last; item += rng.step, ++tcount) {
      const Item w = decode(p, item);
      const int kc0 = w.split * p.kcps;
      const int kc1 = min(p.total_kc, kc0 + p.kcps);
      const int acc = tcount & 1, ra = tcount >> 1;
      int key = -1;
      if (B_RES) {
        key = b_key(p, item);
        if (key != cur_key) {
          ++brun;
          if (!mbar_wait(bfull_bar, brun & 1, p.err, p.wait_ns)) {
            ok = false;
            break;
          }
          cur_key = key;
        }
      }
      if (!mbar_wait(tempty_bar(acc), (ra & 1) ^ 1, p.err, p.wait_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
      for (int kc = kc0; kc < kc1; ++kc, ++it) {
        const int s = it % C::STAGES, r = it / C::STAGES;
        if (!mbar_wait(full_bar(s), r & 1, p.err, p.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = sA + s * C::A_BYTES;
        const uint32_t b_addr = b_addr_of(s, kc - kc0);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint64_t adesc = A_MN ? make_desc(a_addr + kk * 2048, 8192, 1024)
                                      : make_desc(a_addr + kk * 32, 16, 1024);
          const uint64_t bdesc = B_MN ? make_desc(b_addr + kk * 2048, 8192, 1024)
                                      : make_desc(b_addr + kk * 32, 16, 1024);
          umma_bf16(d_tmem, adesc, bdesc, idesc, (kc > kc0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(empty_bar(s));  // frees the A (and ring B) slot once read
      }
      if (!ok) break;
      umma_commit(tfull_bar(acc));  // accumulator ready for the epilogue
      if (B_RES) {
        const int nxt = item + rng.step;
        if (nxt >= rng.last || b_key(p, nxt) != key) umma_commit(bempty_bar);  // B reusable
      }
    }
    // all MMAs issued by this thread complete before TMEM is released
    umma_commit(drain_bar);
    mbar_drain_wait(drain_bar, 0);
  } else if (SIDE && warp >= 2 + kEpiWarps) {
    // ------------------------------------------------------------ side job
    const int st = threadIdx.x - 32 * (2 + kEpiWarps);
    dequant_rows2d(p.side_q, p.side_ldq, p.side_scales, p.side_dst, p.side_ldd, p.side_rows,
                   p.side_cols, (int64_t)blockIdx.x * (32 * kSideWarps) + st,
                   (int64_t)gridDim.x * (32 * kSideWarps));
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    // warp w drains TMEM lane quadrant (w % 4) and column half (w - 2) / 4 of each tile,
    // 64 columns per tcgen05.ld.  Each 32-row piece is converted into this warp's 4 KB
    // staging tile in the 128-byte-swizzled layout (16-byte chunk k of row r sits at chunk
    // k ^ (r % 8)) and written by one TMA tensor store; TMA clips rows beyond the matrix.
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    constexpr int HALF = BN / 2;
    const uint32_t stage = sEpi + (uint32_t)(warp - 2) * 4096u;
    const uint32_t my_row = stage + (uint32_t)lane * 128u;
    const uint32_t sw = (uint32_t)(lane & 7);
    int tcount = 0;
    for (int item = rng.first; item < rng.last; item += rng.step, ++tcount) {
      const Item w = decode(p, item);
      const int acc = tcount & 1, ra = tcount >> 1;
      // one lane waits so that the warp stays converged for the .sync.aligned loads
      int ready = 0;
      if (lane == 0) ready = mbar_wait(tfull_bar(acc), ra & 1, p.err, p.wait_ns) ? 1 : 0;
      ready = __shfl_sync(0xffffffffu, ready, 0);
      if (!ready) break;
      tc_fence_after();
      const int row0 = w.tm * kBM + q * 32;
      const int n0 = w.tn * BN;
      const int ybase = w.split * p.y_per_split + w.bz * p.y_per_bz + row0;
      const int xbase = w.bz * (int)p.d_boff_col + n0;
#pragma unroll 1
      for (int c = half * HALF; c < (half + 1) * HALF; c += 64) {
        uint32_t v[64];
        tmem_ld64(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN + c), v);
        tmem_wait_ld();
        if (n0 + c >= p.N) continue;  // (uniform across the warp)
        if (p.out_f32) {
#pragma unroll
          for (int h = 0; h < 64; h += 32) {  // two 32-column fp32 pieces
            if (lane == 0) bulk_wait_read0();  // the previous store has read the staging tile
            __syncwarp();
#pragma unroll
            for (int k = 0; k < 8; ++k)
              sts128(my_row + (((uint32_t)k ^ sw) << 4), v[h + 4 * k], v[h + 4 * k + 1],
                     v[h + 4 * k + 2], v[h + 4 * k + 3]);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmD, xbase + c + h, ybase, stage);
              bulk_commit();
            }
          }
        } else {
          if (lane == 0) bulk_wait_read0();
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 hh = __floats2bfloat162_rn(__uint_as_float(v[8 * k + 2 * e]),
                                                        __uint_as_float(v[8 * k + 2 * e + 1]));
              o[e] = *reinterpret_cast<uint32_t*>(&hh);
            }
            sts128(my_row + (((uint32_t)k ^ sw) << 4), o[0], o[1], o[2], o[3]);
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmD, xbase + c, ybase, stage);
            bulk_commit();
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(acc));
    }
    if (lane == 0) bulk_wait0();  // every store of this warp has landed before exit
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

bool make_map(CUtensorMap* map, const UmmaOperand& op, int box_rows) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)op.cols, (cuuint64_t)op.rows};
  cuuint64_t strides[1] = {(cuuint64_t)op.ld * 2};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(op.ptr), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int BN, bool A_MN, bool B_MN, bool B_RES, bool SIDE = false>
cudaError_t launch_t(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& md,
                     const Params& p, int grid, const char* family, cudaStream_t s) {
  auto kern = k_umma_gemm<BN, A_MN, B_MN, B_RES, SIDE>;
  constexpr int threads = kThreads + (SIDE ? 32 * kSideWarps : 0);
  static bool attr_done[64] = {false};  // once per device, outside any stream capture
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg<BN, B_RES>::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  begin_launch(family, s);
  const cudaError_t e = launch_pdl(kern, dim3(grid), dim3(threads), Cfg<BN, B_RES>::SMEM_BYTES, s,
                                   ma, mb, md, p);
  end_launch(family, s);
  return e;
}

template <int BN>
cudaError_t launch_bn(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& md,
                      const Params& p, int grid, bool a_mn, bool b_mn, bool b_res,
                      const char* family, cudaStream_t s) {
  if (p.side_rows > 0) {  // the merged-weight GEMMs: A K-major, B either way, B streamed
    if (a_mn || b_res) return cudaErrorInvalidValue;
    if (!b_mn) return launch_t<BN, false, false, false, true>(ma, mb, md, p, grid, family, s);
    return launch_t<BN, false, true, false, true>(ma, mb, md, p, grid, family, s);
  }
  if (b_res) {  // A K-major only
    if (!b_mn) return launch_t<BN, false, false, true>(ma, mb, md, p, grid, family, s);
    return launch_t<BN, false, true, true>(ma, mb, md, p, grid, family, s);
  }
  if (!a_mn && !b_mn) return launch_t<BN, false, false, false>(ma, mb, md, p, grid, family, s);
  if (!a_mn && b_mn) return launch_t<BN, false, true, false>(ma, mb, md, p, grid, family, s);
  if (a_mn && b_mn) return launch_t<BN, true, true, false>(ma, mb, md, p, grid, family, s);
  return launch_t<BN, true, false, false>(ma, mb, md, p, grid, family, s);
}

// Store map of the output: 32-row boxes of 128 bytes (64 bf16 or 32 fp32), 128-byte swizzle.
bool make_out_map(CUtensorMap* map, void* ptr, int64_t rows, int64_t cols, int64_t ld, bool f32) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  const int es = f32 ? 4 : 2;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * es)};
  cuuint32_t box[2] = {(cuuint32_t)(128 / es), 32u};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   ptr, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

int umma_choose_ksplit(int M, int N, int K, int batch) {
  const int BN = (N % 256 == 0) ? 256 : 128;
  const int tiles = ((M + kBM - 1) / kBM) * ((N + BN - 1) / BN) * batch;
  const int total_kc = (K + kBK - 1) / kBK;
  if (total_kc <= 0) return 1;
  const int sms = num_sms();
  int want = 1;
  if (tiles < sms) want = sms / tiles;  // about one wave of items
  int max_split = total_kc / 4;  // at least 4 k-chunks (256 along K) per split
  if (max_split < 1) max_split = 1;
  if (want > max_split) want = max_split;
  const int kcps = (total_kc + want - 1) / want;
  return (total_kc + kcps - 1) / kcps;  // every split non-empty
}

cudaError_t launch_umma_gemm(const UmmaGemm& g, const char* family, cudaStream_t s) {
  if (g.M <= 0 || g.N <= 0 || g.batch <= 0) return cudaSuccess;
  if (gemm_pairs_enabled() && umma_pair_eligible(g)) return launch_umma_gemm_pair(g, family, s);
  if (g.N % 128 != 0) return cudaErrorInvalidValue;
  const int BN = (g.N % 256 == 0) ? 256 : 128;
  CUtensorMap ma, mb;
  if (!make_map(&ma, g.A, g.A.mn_major ? 64 : kBM)) return cudaErrorInvalidValue;
  if (!make_map(&mb, g.B, g.B.mn_major ? 64 : BN)) return cudaErrorInvalidValue;
  Params p;
  p.M = g.M;
  p.N = g.N;
  p.K = g.K;
  p.batch = g.batch;
  p.total_kc = (g.K + kBK - 1) / kBK;
  if (p.total_kc <= 0) return cudaErrorInvalidValue;
  int ks = g.ksplit < 1 ? 1 : g.ksplit;
  if (ks > p.total_kc) ks = p.total_kc;
  p.kcps = (p.total_kc + ks - 1) / ks;
  p.ksplit = (p.total_kc + p.kcps - 1) / p.kcps;
  if (p.ksplit != ks) return cudaErrorInvalidValue;  // caller sized its output for ks splits
  p.tiles_m = (g.M + kBM - 1) / kBM;
  p.tiles_n = (g.N + BN - 1) / BN;
  const long long items = (long long)p.tiles_m * p.tiles_n * p.ksplit * p.batch;
  if (items > 0x7fffffff) return cudaErrorInvalidValue;
  p.num_items = (int)items;
  p.a_boff_mn = (int)g.A.boff_mn;
  p.a_boff_k = (int)g.A.boff_k;
  p.b_boff_mn = (int)g.B.boff_mn;
  p.b_boff_k = (int)g.B.boff_k;
  p.D = g.D;
  p.out_f32 = g.out_f32;
  p.ldd = g.ldd;
  p.d_boff_col = g.d_boff_col;
  p.d_boff = g.d_boff;
  p.d_split = g.d_split;
  p.side_q = g.side_q;
  p.side_ldq = g.side_ldq;
  p.side_scales = g.side_scales;
  p.side_dst = static_cast<__nv_bfloat16*>(g.side_dst);
  p.side_ldd = g.side_ldd;
  p.side_rows = g.side_rows > 0 ? g.side_rows : 0;
  p.side_cols = g.side_cols;
  if (p.side_rows > 0 &&
      (!g.side_q || !g.side_scales || !g.side_dst || g.side_cols <= 0 || g.side_cols % 16 ||
       g.side_ldq % 16 || g.side_ldd % 8 || (reinterpret_cast<uintptr_t>(g.side_q) & 15) ||
       (reinterpret_cast<uintptr_t>(g.side_dst) & 15)))
    return cudaErrorInvalidValue;
  p.err = device_error_flag();
  if (!p.err) return cudaErrorInvalidDevice;  // the bounded waits need the flag
  p.wait_ns = wait_limit_ns();
  // output as a 2-D row-major tensor: batch entries / splits are row offsets (d_boff,
  // d_split multiples of ldd) or column offsets (d_boff_col)
  if (g.ldd <= 0 || g.d_boff % g.ldd != 0 || g.d_split % g.ldd != 0) return cudaErrorInvalidValue;
  p.y_per_bz = (int)(g.d_boff / g.ldd);
  p.y_per_split = (int)(g.d_split / g.ldd);
  const int64_t out_rows = g.d_split ? (int64_t)p.ksplit * (g.d_split / g.ldd)
                                     : (g.d_boff ? (int64_t)g.batch * (g.d_boff / g.ldd) : g.M);
  CUtensorMap md;
  if (!make_out_map(&md, g.D, out_rows, g.d_cols ? g.d_cols : g.ldd, g.ldd, g.out_f32 != 0))
    return cudaErrorInvalidValue;
  int grid = num_sms();
  if (grid > p.num_items) grid = p.num_items;
  // keep B resident when one item's whole B (K <= 256) fits and the items share it
  const bool b_res = !g.A.mn_major && p.kcps <= 4 && p.ksplit == 1 &&
                     p.num_items >= 2 * grid && p.tiles_m >= 2 && p.side_rows == 0;
  if (BN == 256)
    return launch_bn<256>(ma, mb, md, p, grid, g.A.mn_major, g.B.mn_major, b_res, family, s);
  return launch_bn<128>(ma, mb, md, p, grid, g.A.mn_major, g.B.mn_major, b_res, family, s);
}

}  // namespace poetx
