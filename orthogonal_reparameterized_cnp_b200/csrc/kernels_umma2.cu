// tcgen05 GEMM on CTA pairs (cta_group::2) for the merged-weight products of the layer,
// W = V W0'^T and dV = dW W0' (POET-X technical summary section 2.1: the dense W0' product
// of the input-centric layer, the largest contraction of a step).
//
//   D[M x N] = A[M x K] . B[N x K]^T      (bf16 operands, fp32 accumulation in TMEM, bf16 out)
//
// The two CTAs of a cluster compute one 256 x 256 output tile together.  CTA r of the pair
// loads, per 64-wide K chunk, rows [128 r, 128 r + 128) of the tile's A and rows
// [128 r, 128 r + 128) of its B (half of the tile's N) into its own shared memory with
// TMA; the leader CTA (r = 0) issues tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16),
// which reads both CTAs' shared memory and accumulates row half r of the tile in CTA r's
// TMEM.  Per MAC each SM thus loads half the B bytes of the one-CTA kernel (128 x 256
// tiles), and the freed shared memory holds six operand stages instead of four.
//
// Roles (320 threads per CTA, one CTA per SM, persistent over the tiles of its pair):
//   warp 0      TMA producer, both CTAs: waits for its own stage to be free, loads its
//               halves; the completion bytes of both CTAs land on the leader's full barrier
//   warp 1      TMEM allocation (both CTAs, cta_group::2); MMA issue (leader only):
//               waits on its full barrier, issues 4 MMAs per chunk, and its commits arrive on
//               the stage's empty barrier and the accumulator's full barrier of both CTAs
//   warps 2..9  epilogue, both CTAs: tcgen05.ld of the CTA's 128 accumulator rows, bf16,
//               TMA tensor stores; then a remote arrive on the leader's accumulator-empty
//               barrier
// Two TMEM accumulators (2 x 256 columns) let the epilogue of tile t overlap the main loop
// of tile t + 1.  Loads carry no cluster multicast: each CTA loads distinct data.
//
// Int8 merged weight (Q8 instantiation, POET-XQ: the base weight kept in int8 and
// dequantised where it is used): B is read from two bf16 panel buffers of panel_n rows of
// N each.  Panel 0 is dequantised by a short kernel launched just before; the others by two
// extra warps per CTA: panel p + 1 is dequantised (every CTA converts its share, then bumps
// ready[p + 1]) while the MMAs consume panel p; the
// producers wait for ready[p] before loading a tile of panel p, and the leader's epilogue
// counts consumed[p] per finished tile, so panel p + 2 overwrites buffer p & 1 only after
// every tile of panel p has been multiplied.  The full bf16 weight never exists, and the
// conversion (once per weight element) runs beside the MMAs.
//
// Every mbarrier wait is bounded (Params2::wait_ns): on a timeout the waiting role records
// POETX_ERR_TIMEOUT in the device flag and leaves its loop; the CTAs then drain what they can
// observe with short bounded waits, meet at a cluster barrier and free TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "dequant_dev.cuh"
#include "poetx_internal.h"
#include "umma_ptx.cuh"

namespace poetx {
namespace {

constexpr int kPairBM = 128;   // A rows per CTA (256 per pair)
constexpr int kPairBN = 256;   // N of the pair tile (128 B rows per CTA)
constexpr int kPairBK = 64;
constexpr int kPairStages = 6;
constexpr int kPairThreads = 320;
constexpr int kPairEpiWarps = 8;
constexpr int kPairA = kPairBM * kPairBK * 2;            // 16 KB
constexpr int kPairB = (kPairBN / 2) * kPairBK * 2;      // 16 KB
constexpr int kPairRing = kPairStages * (kPairA + kPairB);
constexpr int kPairEpi = kPairEpiWarps * 4096;
constexpr int kPairSmem = 1024 + kPairRing + kPairEpi + 256;
static_assert(kPairSmem <= 227 * 1024, "shared memory per CTA");
constexpr uint32_t kPairTmemCols = 2 * kPairBN;

struct Params2 {
  int M, N, K, total_kc, tiles_m, tiles_n, num_items;
  int* err;
  unsigned long long wait_ns;
  // Q8: int8 weight W0q [rows x ldq] with per-row scales; panels of panel_n along N
  const int8_t* q;
  long long ldq;
  const float* scales;
  __nv_bfloat16* panel[2];
  long long panel_ld;
  int panel_n, npanels;
  int* ready;     // [npanels]: CTAs that finished their share of panel p
  int* consumed;  // [npanels]: tiles of panel p whose MMAs completed
  int group_m;    // tile raster: groups of group_m M-tiles swept over the N-tiles
};

constexpr int kSideWarps2 = 2;

// Tile (tm, tn) of the pair's item-th output tile.  Tiles run through groups of group_m
// M-tiles, N-tile by N-tile inside a group, so the tiles in flight at one time share a few A
// row blocks and B column blocks (both stay in L2).  With the int8 weight (npanels > 0) the
// groups are formed inside each weight panel and the panels follow one another, since the
// pipeline consumes the weight panel by panel.
__device__ __forceinline__ void pair_tile(const Params2& p, int item, int& tm, int& tn) {
  int tn0 = 0, ntn = p.tiles_n, local = item;
  if (p.npanels > 0) {
    const int tpp = p.panel_n / kPairBN;  // N-tiles per full panel
    const int pan = item / (p.tiles_m * tpp);
    tn0 = pan * tpp;
    ntn = min(tpp, p.tiles_n - tn0);
    local = item - pan * p.tiles_m * tpp;
  }
  const int per_group = p.group_m * ntn;
  const int g = local / per_group;
  const int first = g * p.group_m;
  const int gm = min(p.tiles_m - first, p.group_m);
  const int l2 = local - g * per_group;
  tm = first + l2 % gm;
  tn = tn0 + l2 / gm;
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
// the address of this CTA's shared variable `a` in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_to_rank(uint32_t a, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// bounded wait with cluster-scope acquire (barriers that the peer CTA arrives on)
__device__ __noinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, int* err,
                                               unsigned long long limit_ns) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  unsigned spins = 0;
  while (!mbar_try_wait_cluster(bar, parity)) {
    if ((++spins & 63u) == 0) {
      if (*reinterpret_cast<volatile int*>(err) != 0) return false;
      if (globaltimer() - t0 > limit_ns) {
        atomicCAS(err, 0, (int)POETX_ERR_TIMEOUT);
        return false;
      }
    }
  }
  return true;
}
// TMA load into this CTA's shared memory whose completion bytes go to `mbar_cluster`, a
// barrier of either CTA of the pair (no multicast)
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int x, int y,
                                                 uint32_t mbar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(mbar_cluster)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrives once on the barrier at offset `bar` of every CTA in `mask` when all MMAs issued so
// far by this thread have completed
__device__ __forceinline__ void umma_commit_pair_mc(uint32_t bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}
__device__ __forceinline__ void umma_commit_pair(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_gpu(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// orders this thread's generic-proxy global accesses with its async-proxy (TMA) ones
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
// bounded wait until *cnt >= need (acquire)
__device__ __noinline__ bool wait_count(const int* cnt, int need, int* err,
                                        unsigned long long limit_ns) {
  if (ld_acquire_gpu(cnt) >= need) return true;
  const unsigned long long t0 = globaltimer();
  unsigned spins = 0;
  while (ld_acquire_gpu(cnt) < need) {
    if ((++spins & 31u) == 0) {
      if (*reinterpret_cast<volatile int*>(err) != 0) return false;
      if (globaltimer() - t0 > limit_ns) {
        atomicCAS(err, 0, (int)POETX_ERR_TIMEOUT);
        return false;
      }
      __nanosleep(128);
    }
  }
  return true;
}

template <bool B_MN>
__device__ __forceinline__ uint32_t make_idesc_pair() {
  return (1u << 4)                              // D format: f32
         | (1u << 7)                            // A format: bf16
         | (1u << 10)                           // B format: bf16
         | (0u << 15)                           // A K-major
         | ((B_MN ? 1u : 0u) << 16)             // B major
         | ((uint32_t)(kPairBN >> 3) << 17)     // N = 256
         | ((uint32_t)(256 >> 4) << 24);        // M = 256 (the pair)
}

template <bool B_MN, bool Q8>
__global__ void __launch_bounds__(kPairThreads + (Q8 ? 32 * kSideWarps2 : 0), 1)
    k_umma_gemm_pair(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmB1,
                     const __grid_constant__ CUtensorMap tmD, const Params2 p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t sA = base;                                   // stages x 16 KB
  const uint32_t sB = base + kPairStages * kPairA;            // stages x 16 KB
  const uint32_t sEpi = base + kPairRing;                     // 1024-aligned staging tiles
  const uint32_t sBar = sEpi + kPairEpi;
  auto full_bar = [&](int s) { return sBar + 8u * s; };
  auto empty_bar = [&](int s) { return sBar + 8u * (kPairStages + s); };
  auto tfull_bar = [&](int a) { return sBar + 8u * (2 * kPairStages + a); };
  auto tempty_bar = [&](int a) { return sBar + 8u * (2 * kPairStages + 2 + a); };
  const uint32_t drain_bar = sBar + 8u * (2 * kPairStages + 4);
  const uint32_t tmem_slot = sBar + 8u * (2 * kPairStages + 5);
  unsigned char* generic_base = smem_raw + (base - raw);
  volatile uint32_t* tmem_slot_ptr =
      reinterpret_cast<volatile uint32_t*>(generic_base + (tmem_slot - base));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int cid = blockIdx.x >> 1, nclusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 2 * kPairEpiWarps);  // the epilogue warps of both CTAs
    }
    mbar_init(drain_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    if (Q8) prefetch_tmap(&tmB1);
    prefetch_tmap(&tmD);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kPairTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive or TMA completion
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot_ptr;
  pdl_trigger();
  pdl_wait();

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    int it = 0;
    bool ok = true;
    int seen = -1;  // highest panel known to be ready (Q8)
    for (int item = cid; ok && item < p.num_items; item += nclusters) {
      int tm, tn;
      pair_tile(p, item, tm, tn);
      const int m0 = tm * 256 + (int)rank * kPairBM;
      int n0 = tn * kPairBN + (int)rank * (kPairBN / 2);
      const CUtensorMap* mapB = &tmB;
      if (Q8) {
        const int pan = (tn * kPairBN) / p.panel_n;
        if (pan > seen) {
          if (!wait_count(p.ready + pan, (int)gridDim.x, p.err, p.wait_ns)) {
            ok = false;
            break;
          }
          fence_proxy_async_global();  // the panel's generic-proxy writes, then TMA reads
          seen = pan;
        }
        n0 -= pan * p.panel_n;
        mapB = (pan & 1) ? &tmB1 : &tmB;
      }
      for (int kc = 0; kc < p.total_kc; ++kc, ++it) {
        const int s = it % kPairStages, r = it / kPairStages;
        if (!mbar_wait(empty_bar(s), (r & 1) ^ 1, p.err, p.wait_ns)) {
          ok = false;
          break;
        }
        if (leader) mbar_expect_tx(full_bar(s), 2u * (kPairA + kPairB));
        const uint32_t fb = map_to_rank(full_bar(s), 0);
        const int k = kc * kPairBK;
        tma_load_2d_pair(sA + s * kPairA, &tmA, k, m0, fb);
        const uint32_t b_dst = sB + s * kPairB;
        if (!B_MN) {
          tma_load_2d_pair(b_dst, mapB, k, n0, fb);
        } else {
          tma_load_2d_pair(b_dst, mapB, n0, k, fb);
          tma_load_2d_pair(b_dst + 8192, mapB, n0 + 64, k, fb);
        }
      }
    }
    if (!ok && leader) {
      // no TMA write may still be in flight into the leader's stages when it leaves
      const int last = it;
      for (int j = (last > kPairStages ? last - kPairStages : 0); j < last; ++j)
        mbar_drain_wait(full_bar(j % kPairStages), (j / kPairStages) & 1);
    }
  } else if (warp == 1 && lane == 0 && leader) {
    // ------------------------------------------------------------ MMA issuer (leader)
    const uint32_t idesc = make_idesc_pair<B_MN>();
    int it = 0, tcount = 0;
    bool ok = true;
    for (int item = cid; ok && item < p.num_items; item += nclusters, ++tcount) {
      const int acc = tcount & 1, ra = tcount >> 1;
      if (!mbar_wait_cluster(tempty_bar(acc), (ra & 1) ^ 1, p.err, p.wait_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kPairBN);
      for (int kc = 0; kc < p.total_kc; ++kc, ++it) {
        const int s = it % kPairStages, r = it / kPairStages;
        if (!mbar_wait(full_bar(s), r & 1, p.err, p.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = sA + s * kPairA;
        const uint32_t b_addr = sB + s * kPairB;
#pragma unroll
        for (int kk = 0; kk < kPairBK / 16; ++kk) {
          const uint64_t adesc = make_desc(a_addr + kk * 32, 16, 1024);
          const uint64_t bdesc = B_MN ? make_desc(b_addr + kk * 2048, 8192, 1024)
                                      : make_desc(b_addr + kk * 32, 16, 1024);
          umma_bf16_pair(d_tmem, adesc, bdesc, idesc, (kc > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit_pair_mc(empty_bar(s), (uint16_t)0x3);  // both CTAs' stage s is free
      }
      if (!ok) break;
      umma_commit_pair_mc(tfull_bar(acc), (uint16_t)0x3);  // both accumulator halves ready
    }
    // every MMA issued here completes before TMEM is released
    umma_commit_pair(drain_bar);
    mbar_drain_wait(drain_bar, 0);
  } else if (Q8 && warp >= 2 + kPairEpiWarps) {
    // ------------------------------------------------------------ panel dequantisation
    const int st = threadIdx.x - 32 * (2 + kPairEpiWarps);
    for (int pan = 1; pan < p.npanels; ++pan) {  // panel 0 arrives dequantised
      if (pan >= 2) {  // buffer pan & 1 still holds panel pan - 2 until all its tiles ran
        const int cols = min(p.panel_n, p.N - (pan - 2) * p.panel_n);
        const int need = p.tiles_m * (cols / kPairBN);
        if (st == 0) wait_count(p.consumed + pan - 2, need, p.err, p.wait_ns);
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kSideWarps2) : "memory");
        // a failed wait has set the flag: every side thread sees it after the barrier
        if (*reinterpret_cast<volatile int*>(p.err) != 0) break;
        fence_proxy_async_global();
      }
      const int n_first = pan * p.panel_n;
      const int width = min(p.panel_n, p.N - n_first);
      __nv_bfloat16* const dst = (pan & 1) ? p.panel[1] : p.panel[0];
      const int64_t first = (int64_t)blockIdx.x * (32 * kSideWarps2) + st;
      const int64_t stride = (int64_t)gridDim.x * (32 * kSideWarps2);
      if (!B_MN)  // B rows n of W0' (rows of W0q), all K columns
        dequant_rows2d(p.q + (int64_t)n_first * p.ldq, p.ldq, p.scales + n_first, dst, p.panel_ld,
                       width, p.K, first, stride);
      else        // columns n of W0' for every row k of W0q
        dequant_rows2d(p.q + n_first, p.ldq, p.scales, dst, p.panel_ld, p.K, width, first,
                       stride);
      fence_proxy_async_global();
      __threadfence();
      asm volatile("bar.sync 1, %0;" ::"n"(32 * kSideWarps2) : "memory");
      if (st == 0) red_release_gpu(p.ready + pan, 1);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    // warp w drains TMEM lane quadrant (w % 4) and column half (w - 2) / 4 of this CTA's
    // 128 accumulator rows, 64 columns per tcgen05.ld; each 32-row piece goes through the
    // warp's 4 KB 128-byte-swizzled staging tile to a TMA tensor store.
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    constexpr int HALF = kPairBN / 2;
    const uint32_t stage = sEpi + (uint32_t)(warp - 2) * 4096u;
    const uint32_t my_row = stage + (uint32_t)lane * 128u;
    const uint32_t sw = (uint32_t)(lane & 7);
    int tcount = 0;
    for (int item = cid; item < p.num_items; item += nclusters, ++tcount) {
      int tm, tn;
      pair_tile(p, item, tm, tn);
      const int acc = tcount & 1, ra = tcount >> 1;
      int ready = 0;
      if (lane == 0) ready = mbar_wait(tfull_bar(acc), ra & 1, p.err, p.wait_ns) ? 1 : 0;
      ready = __shfl_sync(0xffffffffu, ready, 0);
      if (!ready) break;
      tc_fence_after();
      if (Q8 && leader && warp == 2 && lane == 0)  // the tile's operands are all consumed
        red_release_gpu(p.consumed + (tn * kPairBN) / p.panel_n, 1);
      const int row0 = tm * 256 + (int)rank * kPairBM + q * 32;
      const int n0 = tn * kPairBN;
#pragma unroll 1
      for (int c = half * HALF; c < (half + 1) * HALF; c += 64) {
        uint32_t v[64];
        tmem_ld64(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * kPairBN + c), v);
        tmem_wait_ld();
        if (n0 + c >= p.N) continue;  // (uniform across the warp)
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
          tma_store_2d(&tmD, n0 + c, row0, stage);
          bulk_commit();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(map_to_rank(tempty_bar(acc), 0));
    }
    if (lane == 0) bulk_wait0();  // every store of this warp has landed before exit
    __syncwarp();
  }

  tc_fence_before();
  cluster_sync();  // both CTAs are done with TMEM, shared memory and the barriers
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, kPairTmemCols);
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    tried = true;
  }
  return fn;
}

bool map2d(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols, int64_t ld,
           uint32_t box_cols, uint32_t box_rows, bool store) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             store ? CU_TENSOR_MAP_L2_PROMOTION_NONE : CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool B_MN, bool Q8>
cudaError_t launch_pair_t(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mb1,
                          const CUtensorMap& md, const Params2& p, int grid, const char* family,
                          cudaStream_t s) {
  auto kern = k_umma_gemm_pair<B_MN, Q8>;
  constexpr int threads = kPairThreads + (Q8 ? 32 * kSideWarps2 : 0);
  static bool attr_done[64] = {false};  // once per device, outside any stream capture
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kPairSmem);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = kPairSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  begin_launch(family, s);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ma, mb, mb1, md, p);
  end_launch(family, s);
  return e;
}

// Largest grid (an even number of CTAs) whose clusters are all resident at once: the Q8
// pipeline's CTAs wait for one another's panel shares, so none may wait for a slot.
template <bool B_MN, bool Q8>
int resident_pair_grid() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (cache[dev]) return cache[dev];
  int grid = (num_sms() / 2) * 2;
  if (Q8) {
    auto kern = k_umma_gemm_pair<B_MN, Q8>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kPairSmem) ==
        cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(grid);
      cfg.blockDim = dim3(kPairThreads + 32 * kSideWarps2);
      cfg.dynamicSmemBytes = kPairSmem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int nc = 0;
      if (cudaOccupancyMaxActiveClusters(&nc, kern, &cfg) == cudaSuccess && nc > 0 &&
          2 * nc < grid)
        grid = 2 * nc;
    }
  }
  cache[dev] = grid;
  return grid;
}

}  // namespace

bool umma_pair_eligible(const UmmaGemm& g) {
  return g.batch == 1 && g.ksplit <= 1 && !g.A.mn_major && !g.out_f32 && g.side_rows == 0 &&
         g.N % kPairBN == 0 && g.M >= 256 && g.K >= kPairBK && g.ldd == g.N &&
         (g.d_cols == 0 || g.d_cols == g.N) &&
         g.A.boff_k == 0 && g.A.boff_mn == 0 && g.B.boff_k == 0 && g.B.boff_mn == 0 &&
         g.d_boff == 0 && g.d_boff_col == 0 && g.d_split == 0;
}

static cudaError_t pair_params(const UmmaGemm& g, Params2* p) {
  *p = Params2{};
  p->M = g.M;
  p->N = g.N;
  p->K = g.K;
  p->total_kc = (g.K + kPairBK - 1) / kPairBK;
  p->tiles_m = (g.M + 255) / 256;
  p->tiles_n = g.N / kPairBN;
  const long long items = (long long)p->tiles_m * p->tiles_n;
  if (items > 0x7fffffff) return cudaErrorInvalidValue;
  p->num_items = (int)items;
  p->err = device_error_flag();
  if (!p->err) return cudaErrorInvalidDevice;  // the bounded waits need the flag
  p->wait_ns = wait_limit_ns();
  p->group_m = 8;
  return cudaSuccess;
}

cudaError_t launch_umma_gemm_pair(const UmmaGemm& g, const char* family, cudaStream_t s) {
  if (!umma_pair_eligible(g)) return cudaErrorInvalidValue;
  CUtensorMap ma, mb, md;
  // A K-major: boxes of 128 rows x 64 K.  B K-major: 128 N-rows x 64 K; MN-major: 64 K-rows
  // x 64 N (two per stage).  Output: 32-row boxes of 64 bf16.
  if (!map2d(&ma, g.A.ptr, g.A.rows, g.A.cols, g.A.ld, 64u, (uint32_t)kPairBM, false))
    return cudaErrorInvalidValue;
  if (!map2d(&mb, g.B.ptr, g.B.rows, g.B.cols, g.B.ld, 64u, g.B.mn_major ? 64u : 128u, false))
    return cudaErrorInvalidValue;
  if (!map2d(&md, g.D, g.M, g.N, g.ldd, 64u, 32u, true)) return cudaErrorInvalidValue;
  Params2 p;
  cudaError_t e = pair_params(g, &p);
  if (e != cudaSuccess) return e;
  int grid = (num_sms() / 2) * 2;
  if (grid > 2 * p.num_items) grid = 2 * p.num_items;
  if (grid < 2) return cudaErrorInvalidValue;
  return g.B.mn_major ? launch_pair_t<true, false>(ma, mb, mb, md, p, grid, family, s)
                      : launch_pair_t<false, false>(ma, mb, mb, md, p, grid, family, s);
}

cudaError_t launch_umma_gemm_pair_q8(const UmmaGemm& g, const PairQ8& q, const char* family,
                                     cudaStream_t s) {
  // g.B describes the bf16 merged weight the panels come from (its shape and major-ness);
  // its pointer is not read
  if (!umma_pair_eligible(g) || !q.q || !q.scales || !q.panel[0] || !q.panel[1] ||
      !q.counters || q.panel_n <= 0 || q.panel_n % kPairBN != 0)
    return cudaErrorInvalidValue;
  const bool b_mn = g.B.mn_major != 0;
  const int npan = (g.N + q.panel_n - 1) / q.panel_n;
  // panel layout: K-major B -> [panel_n rows (N) x K], row stride K; MN-major B ->
  // [K rows x panel_n (N)], row stride panel_n
  const int64_t prow = b_mn ? g.K : q.panel_n, pcol = b_mn ? q.panel_n : g.K;
  if (q.ldq % 16 != 0 || pcol % 16 != 0 || (reinterpret_cast<uintptr_t>(q.q) & 15) ||
      (reinterpret_cast<uintptr_t>(q.panel[0]) & 15) || (reinterpret_cast<uintptr_t>(q.panel[1]) & 15))
    return cudaErrorInvalidValue;
  CUtensorMap ma, mb0, mb1, md;
  if (!map2d(&ma, g.A.ptr, g.A.rows, g.A.cols, g.A.ld, 64u, (uint32_t)kPairBM, false))
    return cudaErrorInvalidValue;
  if (!map2d(&mb0, q.panel[0], prow, pcol, pcol, 64u, b_mn ? 64u : 128u, false) ||
      !map2d(&mb1, q.panel[1], prow, pcol, pcol, 64u, b_mn ? 64u : 128u, false))
    return cudaErrorInvalidValue;
  if (!map2d(&md, g.D, g.M, g.N, g.ldd, 64u, 32u, true)) return cudaErrorInvalidValue;
  Params2 p;
  cudaError_t e = pair_params(g, &p);
  if (e != cudaSuccess) return e;
  p.q = q.q;
  p.ldq = q.ldq;
  p.scales = q.scales;
  p.panel[0] = static_cast<__nv_bfloat16*>(q.panel[0]);
  p.panel[1] = static_cast<__nv_bfloat16*>(q.panel[1]);
  p.panel_ld = pcol;
  p.panel_n = q.panel_n;
  p.npanels = npan;
  p.ready = q.counters;
  p.consumed = q.counters + npan;
  const int grid = b_mn ? resident_pair_grid<true, true>() : resident_pair_grid<false, true>();
  if (grid < 2) return cudaErrorInvalidValue;
  // counters: ready[0] = grid (panel 0 is filled below), everything else 0
  e = launch_fill_ints(q.counters, 2 * npan, grid, family, s);
  if (e != cudaSuccess) return e;
  const int w0 = npan > 1 ? q.panel_n : g.N;
  e = b_mn ? launch_dequant_2d(q.q, q.ldq, q.scales, q.panel[0], pcol, g.K, w0, s)
           : launch_dequant_2d(q.q, q.ldq, q.scales, q.panel[0], pcol, w0, g.K, s);
  if (e != cudaSuccess) return e;
  return b_mn ? launch_pair_t<true, true>(ma, mb0, mb1, md, p, grid, family, s)
              : launch_pair_t<false, true>(ma, mb0, mb1, md, p, grid, family, s);
}

}  // namespace poetx
