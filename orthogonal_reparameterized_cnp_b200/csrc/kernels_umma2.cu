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
// Roles (bf16 weight: 320 threads per CTA, one CTA per SM, persistent over the tiles of its
// pair):
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
// dequantised where it is used): warp 0 loads only A (a 4-stage ring); one more warp loads
// each CTA's B tile as int8 codes (8 KB per K chunk, half the bytes of bf16) into staging
// slots, and four groups of two converter warps turn the codes into bf16(s * q) (fp32
// product, round to nearest even, the scale s of the code's row of W0'), written straight
// into a 4-stage ring of B operands in the 128-byte-swizzled layout the MMA reads.  The MMA
// waits for both rings and frees both; four epilogue warps (instead of eight) drain TMEM.
// No bf16 copy of the weight exists in global memory, and the operands equal those of the
// bf16 kernel on the dequantised weight, so the results are the same bit for bit.  Measured
// rate: about 0.8 of the bf16 kernel's.  More converter warps, deeper rings, converters
// reading the codes straight from global memory (less shared-memory traffic) and a 512 x 128
// pair tile (half the conversions per FLOP, more shared-memory traffic) did not raise it.
//
// Every mbarrier wait is bounded (Params2::wait_ns): on a timeout the waiting role records
// POETX_ERR_TIMEOUT in the device flag and leaves its loop; the CTAs then drain what they can
// observe with short bounded waits, meet at a cluster barrier and free TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "poetx_internal.h"
#include "umma_ptx.cuh"

namespace poetx {
namespace {

constexpr int kPairBM = 128;   // A rows per CTA (256 per pair)
constexpr int kPairBN = 256;   // N of the pair tile (128 B rows per CTA)
constexpr int kPairBK = 64;
constexpr int kPairA = kPairBM * kPairBK * 2;            // 16 KB
constexpr int kPairB = (kPairBN / 2) * kPairBK * 2;      // 16 KB
constexpr int kQ8Bytes = (kPairBN / 2) * kPairBK;        // 8 KB: one CTA's int8 B tile
#ifndef PAIR_Q8_GROUPS
#define PAIR_Q8_GROUPS 4
#endif
#ifndef PAIR_Q8_GROUP_WARPS
#define PAIR_Q8_GROUP_WARPS 2
#endif
#ifndef PAIR_Q8_EPI
#define PAIR_Q8_EPI 4
#endif
// int8 weight: converter group g (kGroupWarps warps) owns the K chunks it = g (mod G) of the
// CTA's flat chunk sequence and staging slots 2 g, 2 g + 1 (used in turn)
constexpr int kConvGroups = PAIR_Q8_GROUPS;
constexpr int kGroupWarps = PAIR_Q8_GROUP_WARPS;
constexpr int kConvWarps = kConvGroups * kGroupWarps;
constexpr int kGroupThreads = 32 * kGroupWarps;
constexpr int kTileChunks = kQ8Bytes / 16;                 // 16-code chunks per int8 tile
constexpr int kConvChunks = (kTileChunks + kGroupThreads - 1) / kGroupThreads;  // per thread

// Per instantiation: RA stages of A and RB stages of B (with the bf16 weight one ring that
// TMA fills; with the int8 weight A's stages are filled by TMA and B's by the converters, each
// with barriers of its own, and four of each leave room for the staging slots), epilogue
// warps, staging slots, threads and shared memory.
template <bool Q8>
struct PairCfg {
  static constexpr int RA = Q8 ? 4 : 6;
  static constexpr int RB = Q8 ? 4 : 6;
  static constexpr int EPI = Q8 ? PAIR_Q8_EPI : 8;
  static constexpr bool ld32 = Q8 && kConvWarps > 8;  // epilogue loads of 32 columns
  static constexpr int SLOTS = Q8 ? 2 * kConvGroups : 0;
  static constexpr int threads = 64 + 32 * EPI + (Q8 ? 32 + 32 * kConvWarps : 0);
  // with the int8 weight and RA == RB one set of stage barriers serves both operands
  static constexpr bool split = Q8 && RA != RB;
  static constexpr int nbar = 2 * RA + (split ? 2 * RB : 0) + 6 + 2 * SLOTS;
  static constexpr int smem =
      1024 + RA * kPairA + RB * kPairB + SLOTS * kQ8Bytes + EPI * 4096 + 512;
};
static_assert(PairCfg<false>::smem <= 227 * 1024 && PairCfg<true>::smem <= 227 * 1024,
              "shared memory per CTA");
static_assert(PairCfg<false>::nbar * 8 <= 512 && PairCfg<true>::nbar * 8 <= 512, "barriers");
// a group's waits on the converted-operand ring see consecutive phases
static_assert(kConvGroups <= PairCfg<true>::RB, "converter groups");
static_assert(PairCfg<true>::threads <= 1024, "threads");
constexpr uint32_t kPairTmemCols = 2 * kPairBN;

#ifndef PAIR_GROUP_M
#define PAIR_GROUP_M 8  // M-tiles per raster group
#endif
struct Params2 {
  int M, N, K, total_kc, tiles_m, tiles_n, num_items;
  int* err;
  unsigned long long wait_ns;
  const float* scales;  // Q8: scale of each row of the int8 weight
  int group_m;          // tile raster: groups of group_m M-tiles swept over the N-tiles
};

// Tile (tm, tn) of the pair's item-th output tile.  Tiles run through groups of group_m
// M-tiles, N-tile by N-tile inside a group, so the tiles in flight at one time share a few A
// row blocks and B column blocks (both stay in L2).
__device__ __forceinline__ void pair_tile(const Params2& p, int item, int& tm, int& tn) {
  const int per_group = p.group_m * p.tiles_n;
  const int g = item / per_group;
  const int first = g * p.group_m;
  const int gm = min(p.tiles_m - first, p.group_m);
  const int l2 = item - g * per_group;
  tm = first + l2 % gm;
  tn = l2 / gm;
}

// 16 int8 codes q (one 16-byte chunk) -> 16 bf16 values bf16(s * q) in o[0..7] (element e in
// the low half of o[e / 2] when e is even).  Byte b of (word ^ 0x80808080) is q + 128; put
// under the exponent of 2^23 it is the float 2^23 + q + 128, and subtracting 2^23 + 128
// leaves q exactly.  The product s * q is one fp32 multiply rounded to nearest even, then
// rounded to bf16 (nearest even) - the same value as the dequantisation kernel writes.
#ifndef PAIR_Q8_F32X2
#define PAIR_Q8_F32X2 1
#endif
__device__ __forceinline__ void q8_chunk_to_bf16(const uint4 w, float s, uint32_t (&o)[8]) {
  const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t u = words[i] ^ 0x80808080u;
#if PAIR_Q8_F32X2
    // the same operations two lanes at a time (packed fp32 add and multiply, each lane
    // rounded to nearest even)
    uint32_t e[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) e[b] = __byte_perm(u, 0x4B000000u, 0x7440u + (uint32_t)b);
    const unsigned long long off = ((unsigned long long)__float_as_uint(8388736.0f) << 32) |
                                   __float_as_uint(8388736.0f);
    const unsigned long long sc2 = ((unsigned long long)__float_as_uint(s) << 32) |
                                   __float_as_uint(s);
    unsigned long long v01 = ((unsigned long long)e[1] << 32) | e[0];
    unsigned long long v23 = ((unsigned long long)e[3] << 32) | e[2];
    asm("sub.rn.f32x2 %0, %0, %1;" : "+l"(v01) : "l"(off));
    asm("sub.rn.f32x2 %0, %0, %1;" : "+l"(v23) : "l"(off));
    asm("mul.rn.f32x2 %0, %0, %1;" : "+l"(v01) : "l"(sc2));
    asm("mul.rn.f32x2 %0, %0, %1;" : "+l"(v23) : "l"(sc2));
    __nv_bfloat162 lo = __floats2bfloat162_rn(__uint_as_float((uint32_t)v01),
                                              __uint_as_float((uint32_t)(v01 >> 32)));
    __nv_bfloat162 hi = __floats2bfloat162_rn(__uint_as_float((uint32_t)v23),
                                              __uint_as_float((uint32_t)(v23 >> 32)));
#else
    float f[4];
#pragma unroll
    for (int b = 0; b < 4; ++b)
      f[b] = __fsub_rn(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7440u + (uint32_t)b)),
                       8388736.0f);
    __nv_bfloat162 lo = __floats2bfloat162_rn(__fmul_rn(s, f[0]), __fmul_rn(s, f[1]));
    __nv_bfloat162 hi = __floats2bfloat162_rn(__fmul_rn(s, f[2]), __fmul_rn(s, f[3]));
#endif
    o[2 * i] = *reinterpret_cast<uint32_t*>(&lo);
    o[2 * i + 1] = *reinterpret_cast<uint32_t*>(&hi);
  }
}
// MN-major int8 tile (64 K rows of 8 chunks of 16 codes): chunk index ch -> (K row kr, chunk
// c).  Each run of 16 indices covers two rows; its first 8 take chunks 0-3 of the first row
// and 4-7 of the second, the next 8 the other halves.  Any 8 consecutive indices then read 8
// different 16-byte bank groups of the staging tile (c differs) and write 8 different ones
// of the two operand boxes (box c / 4 of either row, whose swizzles differ in bit 0).
__device__ __forceinline__ void mn_chunk(int ch, int& kr, int& c) {
  const int j = ch & 15, half = j >> 3, i = j & 7;
  kr = 2 * (ch >> 4) + (i >> 2);
  c = (i & 3) | ((((i >> 2) ^ half) & 1) << 2);
}

// AND of v over the `count` threads meeting at named barrier `id`
__device__ __forceinline__ bool group_all(bool v, int id, int count) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.cta.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void named_sync(int id, int count) {
  asm volatile("barrier.cta.sync.aligned %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
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

// tmB: the bf16 B operand, or (Q8) the int8 weight W0q with 8 KB boxes and no swizzle
template <bool B_MN, bool Q8>
__global__ void __launch_bounds__(PairCfg<Q8>::threads, 1)
    k_umma_gemm_pair(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmD, const Params2 p) {
  using C = PairCfg<Q8>;
  constexpr int RA = C::RA, RB = C::RB, EPI = C::EPI;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t sA = base;                                   // RA x 16 KB
  const uint32_t sB = sA + RA * kPairA;                       // RB x 16 KB
  const uint32_t sQ = sB + RB * kPairB;                       // Q8: slots x 8 KB
  const uint32_t sEpi = sQ + C::SLOTS * kQ8Bytes;             // 1024-aligned staging tiles
  const uint32_t sBar = sEpi + EPI * 4096;
  // A ring (with the bf16 weight: the common ring of A and B)
  auto fullA = [&](int s) { return sBar + 8u * s; };
  auto emptyA = [&](int s) { return sBar + 8u * (RA + s); };
  // Q8: ring of converted B operands (the A ring's barriers when the rings are equal)
  auto fullB = [&](int s) { return C::split ? sBar + 8u * (2 * RA + s) : fullA(s); };
  auto emptyB = [&](int s) { return C::split ? sBar + 8u * (2 * RA + RB + s) : emptyA(s); };
  constexpr int X = 2 * RA + (C::split ? 2 * RB : 0);
  auto tfull_bar = [&](int a) { return sBar + 8u * (X + a); };
  auto tempty_bar = [&](int a) { return sBar + 8u * (X + 2 + a); };
  const uint32_t drain_bar = sBar + 8u * (X + 4);
  const uint32_t tmem_slot = sBar + 8u * (X + 5);
  auto q8full_bar = [&](int j) { return sBar + 8u * (X + 6 + j); };
  auto q8free_bar = [&](int j) { return sBar + 8u * (X + 6 + C::SLOTS + j); };
  unsigned char* generic_base = smem_raw + (base - raw);
  volatile uint32_t* tmem_slot_ptr =
      reinterpret_cast<volatile uint32_t*>(generic_base + (tmem_slot - base));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int cid = blockIdx.x >> 1, nclusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < RA; ++s) {
      // the leader's expect_tx (and the TMA bytes of both CTAs); with shared stage barriers
      // also one arrival from the owning converter group of each CTA
      mbar_init(fullA(s), (Q8 && !C::split) ? 3 : 1);
      mbar_init(emptyA(s), 1);
    }
    if (Q8) {
      if (C::split) {
        for (int s = 0; s < RB; ++s) {
          mbar_init(fullB(s), 2);  // the owning converter group of each CTA
          mbar_init(emptyB(s), 1);
        }
      }
      for (int j = 0; j < C::SLOTS; ++j) {
        mbar_init(q8full_bar(j), 1);
        mbar_init(q8free_bar(j), 1);
      }
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 2 * EPI);  // the epilogue warps of both CTAs
    }
    mbar_init(drain_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
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
    for (int item = cid; ok && item < p.num_items; item += nclusters) {
      int tm, tn;
      pair_tile(p, item, tm, tn);
      const int m0 = tm * 256 + (int)rank * kPairBM;
      const int n0 = tn * kPairBN + (int)rank * (kPairBN / 2);
      for (int kc = 0; kc < p.total_kc; ++kc, ++it) {
        const int s = it % RA, r = it / RA;
        if (!mbar_wait(emptyA(s), (r & 1) ^ 1, p.err, p.wait_ns)) {
          ok = false;
          break;
        }
        const uint32_t fb = map_to_rank(fullA(s), 0);
        const int k = kc * kPairBK;
        if (!Q8) {
          if (leader) mbar_expect_tx(fullA(s), 2u * (kPairA + kPairB));
          tma_load_2d_pair(sA + s * kPairA, &tmA, k, m0, fb);
          const uint32_t b_dst = sB + s * kPairB;
          if (!B_MN) {
            tma_load_2d_pair(b_dst, &tmB, k, n0, fb);
          } else {
            tma_load_2d_pair(b_dst, &tmB, n0, k, fb);
            tma_load_2d_pair(b_dst + 8192, &tmB, n0 + 64, k, fb);
          }
        } else {  // A only: the converter groups fill the B ring
          if (leader) mbar_expect_tx(fullA(s), 2u * kPairA);
          tma_load_2d_pair(sA + s * kPairA, &tmA, k, m0, fb);
        }
      }
    }
    if (!ok) {
      // no TMA write may still be in flight into this CTA's shared memory when it leaves
      const int last = it;
      if (leader)
        for (int j = (last > RA ? last - RA : 0); j < last; ++j)
          mbar_drain_wait(fullA(j % RA), (j / RA) & 1);
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
        const int s = it % RA, r = it / RA;
        const int sb = Q8 ? it % RB : s;
        // (converter arrivals come from both CTAs: cluster-scope acquire)
        if (!(Q8 && !C::split ? mbar_wait_cluster(fullA(s), r & 1, p.err, p.wait_ns)
                              : mbar_wait(fullA(s), r & 1, p.err, p.wait_ns)) ||
            (C::split && !mbar_wait_cluster(fullB(sb), (it / RB) & 1, p.err, p.wait_ns))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = sA + s * kPairA;
        const uint32_t b_addr = sB + sb * kPairB;
#pragma unroll
        for (int kk = 0; kk < kPairBK / 16; ++kk) {
          const uint64_t adesc = make_desc(a_addr + kk * 32, 16, 1024);
          const uint64_t bdesc = B_MN ? make_desc(b_addr + kk * 2048, 8192, 1024)
                                      : make_desc(b_addr + kk * 32, 16, 1024);
          umma_bf16_pair(d_tmem, adesc, bdesc, idesc, (kc > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit_pair_mc(emptyA(s), (uint16_t)0x3);  // both CTAs' stage s is free
        if (C::split) umma_commit_pair_mc(emptyB(sb), (uint16_t)0x3);
      }
      if (!ok) break;
      umma_commit_pair_mc(tfull_bar(acc), (uint16_t)0x3);  // both accumulator halves ready
    }
    // every MMA issued here completes before TMEM is released
    umma_commit_pair(drain_bar);
    mbar_drain_wait(drain_bar, 0);
  } else if (Q8 && warp == 2 + EPI) {
    // ------------------------------------------------------------ int8 tile loads
    // The CTA's K chunks form one flat sequence it = (item round) * total_kc + kc.  Chunk
    // it (turn u = it / G of group it % G) goes to slot 2 (it % G) + (u & 1) as soon as the
    // group has converted the slot's previous tile: up to 2 G chunks ahead of the
    // conversions.
    if (lane == 0) {
      const int total = ((p.num_items - cid + nclusters - 1) / nclusters) * p.total_kc;
      int ir = 0, kc = 0, n0 = 0, last_ir = -1;
      int it = 0;
      bool ok = true;
      for (; it < total; ++it) {
        if (ir != last_ir) {
          int tm, tn;
          pair_tile(p, cid + ir * nclusters, tm, tn);
          n0 = tn * kPairBN + (int)rank * (kPairBN / 2);
          last_ir = ir;
        }
        const int u = it / kConvGroups;
        const int slot = 2 * (it % kConvGroups) + (u & 1);
        if (!mbar_wait(q8free_bar(slot), ((u >> 1) & 1) ^ 1, p.err, p.wait_ns)) {
          ok = false;
          break;
        }
        mbar_expect_tx(q8full_bar(slot), (uint32_t)kQ8Bytes);
        const int k = kc * kPairBK;
        if (!B_MN)
          tma_load_2d(sQ + slot * kQ8Bytes, &tmB, k, n0, q8full_bar(slot));
        else
          tma_load_2d(sQ + slot * kQ8Bytes, &tmB, n0, k, q8full_bar(slot));
        if (++kc == p.total_kc) {
          kc = 0;
          ++ir;
        }
      }
      if (!ok) {
        // no int8 load may still be in flight into this CTA's shared memory when it leaves
        for (int j = (it > C::SLOTS ? it - C::SLOTS : 0); j < it; ++j) {
          const int u = j / kConvGroups;
          mbar_drain_wait(q8full_bar(2 * (j % kConvGroups) + (u & 1)), (u >> 1) & 1);
        }
      }
    }
  } else if (Q8 && warp > 2 + EPI) {
    // ------------------------------------------------------------ int8 -> bf16 operands
    // Group g takes chunks it = g + G u (u = 0, 1, ...): it waits for the chunk's int8 tile
    // (slot 2 g + (u & 1)) and for B stage it % RB to be free, converts, completes the stage with one
    // arrival per CTA on the leader's fullB barrier, and frees the slot.
    //
    // Each 8 KB tile is 512 chunks of 16 codes; group thread gt converts chunks gt +
    // kGroupThreads * jj.  K-major B (forward): staging rows are N rows of 64 codes (chunk
    // ch = 4 n + c), and row n of the operand is 128 bytes with 16-byte chunk c stored at
    // c ^ (n & 7).  MN-major B (backward): staging rows are K rows of 128 codes (N), chunk ch
    // mapped to (row, chunk) by mn_chunk, and the operand is two boxes (N 0-63, 64-127) of 64
    // K rows of 128 bytes, chunk c of row k stored at c ^ (k & 7).  In both layouts every 8
    // lanes of a warp load from 8 different bank groups and store to 8 different ones.
    const int cw = threadIdx.x - 32 * (3 + EPI);
    const int grp = cw / kGroupThreads, gt = cw % kGroupThreads;
    const int bar_id = 1 + grp;  // named barrier of the group
    const int total = ((p.num_items - cid + nclusters - 1) / nclusters) * p.total_kc;
    // chunks it = grp, grp + G, ... without divisions: item round ir, K chunk kc, and the
    // operand row n0 of the round's tile (this CTA's half of its N)
    int it = grp, ir = grp / p.total_kc, kc = grp - ir * p.total_kc;
    auto tile_n0 = [&](int r) {
      int tm, tn;
      pair_tile(p, cid + r * nclusters, tm, tn);
      return tn * kPairBN + (int)rank * (kPairBN / 2);
    };
    int n0 = it < total ? tile_n0(ir) : 0;
    int scale_n0 = -1;
    float sc[kConvChunks];
    bool ok = true;
    for (int u = 0; it < total; ++u) {
      const int k = kc * kPairBK;
      if (!B_MN) {  // the scale follows the operand row n: fixed while the tile is
        if (n0 != scale_n0) {
#pragma unroll
          for (int jj = 0; jj < kConvChunks; ++jj) {
            const int ch = gt + kGroupThreads * jj;
            sc[jj] = ch < kTileChunks ? __ldg(p.scales + n0 + (ch >> 2)) : 0.f;
          }
          scale_n0 = n0;
        }
      } else {      // the scale follows the K row
#pragma unroll
        for (int jj = 0; jj < kConvChunks; ++jj) {
          int kr, c;
          mn_chunk(gt + kGroupThreads * jj, kr, c);
          const int o = k + kr;
          // rows past K hold zero codes
          sc[jj] = (o < p.K && gt + kGroupThreads * jj < kTileChunks) ? __ldg(p.scales + o) : 0.f;
        }
      }
      const int sb = it % RB, slot = 2 * grp + (u & 1);
      int got = 1;
      if (lane == 0) {
        got = mbar_wait(q8full_bar(slot), (u >> 1) & 1, p.err, p.wait_ns) &&
              mbar_wait(emptyB(sb), ((it / RB) & 1) ^ 1, p.err, p.wait_ns);
      }
      // every thread of the group takes the same branch (a failed wait of any warp)
      if (!group_all(__shfl_sync(0xffffffffu, got, 0) != 0, bar_id, kGroupThreads)) {
        ok = false;
        break;
      }
      // both phases have completed: every lane acquires them (returns at once)
      while (!mbar_try_wait(q8full_bar(slot), (u >> 1) & 1)) {
      }
      while (!mbar_try_wait(emptyB(sb), ((it / RB) & 1) ^ 1)) {
      }
      const uint32_t src = sQ + slot * kQ8Bytes;
      const uint32_t dst = sB + sb * kPairB;
#pragma unroll
      for (int jj = 0; jj < kConvChunks; ++jj) {
        const int ch = gt + kGroupThreads * jj;
        if (kTileChunks % kGroupThreads != 0 && ch >= kTileChunks) break;
        uint32_t o[8];
        uint32_t row, c0, c1;
        if (!B_MN) {
          q8_chunk_to_bf16(lds128(src + ch * 16), sc[jj], o);
          const uint32_t n = (uint32_t)ch >> 2, c = (uint32_t)ch & 3u;
          row = dst + n * 128u;
          c0 = (2u * c) ^ (n & 7u);
          c1 = (2u * c + 1u) ^ (n & 7u);
        } else {
          int kr_, c_;
          mn_chunk(ch, kr_, c_);
          const uint32_t kr = (uint32_t)kr_, c = (uint32_t)c_;
          q8_chunk_to_bf16(lds128(src + (kr * 8u + c) * 16u), sc[jj], o);
          row = dst + (c >> 2) * 8192u + kr * 128u;
          c0 = (2u * (c & 3u)) ^ (kr & 7u);
          c1 = (2u * (c & 3u) + 1u) ^ (kr & 7u);
        }
        sts128(row + (c0 << 4), o[0], o[1], o[2], o[3]);
        sts128(row + (c1 << 4), o[4], o[5], o[6], o[7]);
      }
      fence_async_smem();  // the generic-proxy stores, then the tensor core's reads
      named_sync(bar_id, kGroupThreads);  // the whole tile is written and the slot read
      if (gt == 0) {
        // The stores are complete in this CTA's shared memory (each thread's proxy fence,
        // then the group barrier) before this arrival is performed, and the leader issues
        // the MMAs that read them only after it observes the phase.  A CTA-scope release is
        // enough for that and costs far less than a cluster-scope one.
        const uint32_t fb = map_to_rank(fullB(sb), 0);
        asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(fb) : "memory");
        mbar_arrive(q8free_bar(slot));  // the slot may be reloaded
      }
      // next chunk of the group
      it += kConvGroups;
      kc += kConvGroups;
      if (kc >= p.total_kc) {
        while (kc >= p.total_kc) {
          kc -= p.total_kc;
          ++ir;
        }
        if (it < total) n0 = tile_n0(ir);
      }
    }
    (void)ok;
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    // warp w drains TMEM lane quadrant (w % 4) and, with 8 epilogue warps, column half
    // (w - 2) / 4 of this CTA's 128 accumulator rows (with 4, all 256 columns), 64 columns per
    // tcgen05.ld; each 32-row piece goes through the warp's 4 KB 128-byte-swizzled staging
    // tile to a TMA tensor store.
    const int q = warp & 3;
    constexpr int COLS = kPairBN / (EPI / 4);
    const int c_first = ((warp - 2) >> 2) * COLS;
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
      const int row0 = tm * 256 + (int)rank * kPairBM + q * 32;
      const int n0 = tn * kPairBN;
#pragma unroll 1
      for (int c = c_first; c < c_first + COLS; c += 64) {
        if (n0 + c >= p.N) continue;  // (uniform across the warp)
        if (lane == 0) bulk_wait_read0();  // the staging tile's previous store has read it
        __syncwarp();
        // 64 columns per tcgen05.ld, or two loads of 32 where registers are short (many
        // converter warps)
#pragma unroll
        for (int h = 0; h < (C::ld32 ? 2 : 1); ++h) {
          constexpr int W = C::ld32 ? 32 : 64;
          uint32_t v[W];
          const uint32_t ta =
              tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * kPairBN + c + h * W);
          if constexpr (W == 32)
            tmem_ld32(ta, v);
          else
            tmem_ld64(ta, v);
          tmem_wait_ld();
#pragma unroll
          for (int kk = 0; kk < W / 8; ++kk) {
            const int k = h * (W / 8) + kk;
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 hh = __floats2bfloat162_rn(__uint_as_float(v[8 * kk + 2 * e]),
                                                        __uint_as_float(v[8 * kk + 2 * e + 1]));
              o[e] = *reinterpret_cast<uint32_t*>(&hh);
            }
            sts128(my_row + (((uint32_t)k ^ sw) << 4), o[0], o[1], o[2], o[3]);
          }
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
cudaError_t launch_pair_t(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& md,
                          const Params2& p, int grid, const char* family, cudaStream_t s) {
  auto kern = k_umma_gemm_pair<B_MN, Q8>;
  constexpr int threads = PairCfg<Q8>::threads;
  constexpr int smem = PairCfg<Q8>::smem;
  static bool attr_done[64] = {false};  // once per device, outside any stream capture
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
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
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ma, mb, md, p);
  end_launch(family, s);
  return e;
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
  p->group_m = PAIR_GROUP_M;
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
  return g.B.mn_major ? launch_pair_t<true, false>(ma, mb, md, p, grid, family, s)
                      : launch_pair_t<false, false>(ma, mb, md, p, grid, family, s);
}

cudaError_t launch_umma_gemm_pair_q8(const UmmaGemm& g, const PairQ8& q, const char* family,
                                     cudaStream_t s) {
  // g.B describes the bf16 merged weight that the codes stand for (its shape and
  // major-ness); its pointer is not read
  if (!umma_pair_eligible(g) || !q.q || !q.scales) return cudaErrorInvalidValue;
  const bool b_mn = g.B.mn_major != 0;
  // W0q [rows x ldq]: K-major B -> rows index N and columns K; MN-major B -> rows index K
  const int64_t rows = b_mn ? g.K : g.N, cols = b_mn ? g.N : g.K;
  if (q.ldq % 16 != 0 || q.ldq < cols || (reinterpret_cast<uintptr_t>(q.q) & 15))
    return cudaErrorInvalidValue;
  auto enc = encode_fn();
  if (!enc) return cudaErrorInvalidValue;
  CUtensorMap ma, mq, md;
  if (!map2d(&ma, g.A.ptr, g.A.rows, g.A.cols, g.A.ld, 64u, (uint32_t)kPairBM, false))
    return cudaErrorInvalidValue;
  {
    // one CTA's int8 tile: 128 N rows x 64 K codes, or 64 K rows x 128 N codes
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)q.ldq};
    cuuint32_t box[2] = {b_mn ? 128u : 64u, b_mn ? 64u : 128u};
    cuuint32_t estr[2] = {1u, 1u};
    if (enc(&mq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(q.q), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  if (!map2d(&md, g.D, g.M, g.N, g.ldd, 64u, 32u, true)) return cudaErrorInvalidValue;
  Params2 p;
  cudaError_t e = pair_params(g, &p);
  if (e != cudaSuccess) return e;
  p.scales = q.scales;
  int grid = (num_sms() / 2) * 2;
  if (grid > 2 * p.num_items) grid = 2 * p.num_items;
  if (grid < 2) return cudaErrorInvalidValue;
  return b_mn ? launch_pair_t<true, true>(ma, mq, md, p, grid, family, s)
              : launch_pair_t<false, true>(ma, mq, md, p, grid, family, s);
}

}  // namespace poetx
