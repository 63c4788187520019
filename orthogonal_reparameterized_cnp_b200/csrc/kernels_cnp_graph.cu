// The Cayley-Neumann parameterisation (POET-X technical summary, section 2.4) as one
// persistent kernel per call: all of a call's steps -- expanding theta into Q, the
// structured fp32 products, the symmetrising combinations, packing dtheta -- are jobs of
// one launch.  Work items (one output tile of one job for one b x b block) are handed
// out in job order through an atomic ticket; before computing, an item waits until the
// jobs it reads have finished for its own block (per-(job, block) counters), so the
// blocks flow through the chain independently and no launch boundary separates steps.
//
// Two shapes of product item:
//   * 64 x 64 output tiles, 512 threads, K split over four 128-thread groups whose partial
//     tiles are summed through shared memory in a fixed order; one CTA per SM.  Used when
//     the call has few blocks (a level of the chain then still has ~one item per SM).
//   * 128 x 128 output tiles, 256 threads, one 8 x 8 register tile per thread over the
//     whole K (no partial-tile reduction), structured epilogue straight from registers;
//     two CTAs per SM, so one CTA's operand waits and epilogue overlap the other's FMAs.
//     Used when the call has enough blocks to fill the GPU with these larger items.
// The elementwise jobs work on 64 x 64 tile pairs in both.
//
// Deadlock freedom: tickets are taken in increasing order by CTAs that are running, and
// an item only waits on items with smaller tickets, so the lowest unfinished ticket can
// always run (the grid is also sized to the CTAs that fit on the GPU at once).  Every wait is bounded anyway: after the
// time limit the CTA records POETX_ERR_TIMEOUT in the device flag and stops.
//
// Data produced inside the launch is read through L2 only (cp.async.cg, ld.global.cg),
// never through the non-coherent L1 / read-only paths.
#include <cuda_bf16.h>

#include "poetx_internal.h"

namespace poetx {
namespace {

// ---- 64 x 64 items ------------------------------------------------------------------
// kGroups groups of 128 threads per CTA; in a product tile every group accumulates the
// whole 64 x 64 tile over its own share of K (own cp.async ring), then the partial tiles
// are summed through shared memory in a fixed order.
constexpr int kGroups = 4;
constexpr int kThreads = kGroups * 128;
constexpr int kGThreads = 128;
constexpr int kBK = 16;
constexpr int kLD = 64 + 4;
constexpr int kStages = 4;
constexpr int kStageFloats = 2 * kBK * kLD;
constexpr int kRingFloats = kGroups * kStages * kStageFloats;  // 139 KB
constexpr int kRedFloats = kGroups * 64 * 64;                   // partial tiles
constexpr int kMirFloats = 2 * 64 * 65;                         // mirror staging
constexpr int kPairFloats = 4 * 64 * 65;  // symmetrising job: 2 inputs x tiles (I,J), (J,I)
// Epilogue operand tiles (the adds and the skew term of a product) are fetched with the
// first k tiles into their own region after the ring, so the epilogue never waits on
// L2.  Row stride 68 keeps 16-byte cp.async destinations.
constexpr int kEpiTiles = 2;
constexpr int kELD = 68;
constexpr int kEpiFloats = kEpiTiles * 64 * kELD;
constexpr int kSmemFloats = kRingFloats + kEpiFloats;
static_assert(kRedFloats + kMirFloats <= kRingFloats,
              "partial tiles and mirror staging must fit in the ring region");
static_assert(kPairFloats <= kSmemFloats, "symmetrising job staging must fit");
constexpr int kSmemBytes = kSmemFloats * 4;
static_assert(kSmemBytes + 1024 <= 227 * 1024, "shared memory per SM");
constexpr int kPT = 64, kPLD = 65;  // 64 x 64 tile-pair jobs

// ---- 128 x 128 items ----------------------------------------------------------------
// Tuning knobs (defaults measured best on B200): k slice depth, cp.async stages, unrolling
// of the k steps of a slice, CTAs per SM, register double-buffering of the operand
// fragments (scalar FMAs only), packed-pair FMAs.
#ifndef CNP2_BK
#define CNP2_BK 32
#endif
#ifndef CNP2_STAGES
#define CNP2_STAGES 3
#endif
#ifndef CNP2_KUNROLL
#define CNP2_KUNROLL CNP2_BK
#endif
#ifndef CNP2_CTAS
#define CNP2_CTAS 2
#endif
#ifndef CNP2_DBUF
#define CNP2_DBUF 0
#endif
#ifndef CNP2_FMA2
#define CNP2_FMA2 1
#endif
#ifndef CNP2_DIAGSKIP
#define CNP2_DIAGSKIP 1
#endif
constexpr int k2Threads = 256;  // 16 x 16 threads, 8 x 8 outputs each
constexpr int k2BK = CNP2_BK;
constexpr int k2LD = 128 + 4;  // row stride of a staged k slice (16-byte aligned rows)
constexpr int k2Stages = CNP2_STAGES;
constexpr int k2KUnroll = CNP2_KUNROLL;
constexpr int k2StageFloats = 2 * k2BK * k2LD;
constexpr int k2RingFloats = k2Stages * k2StageFloats;  // 99 KB
// epilogue operands (the adds and the skew term, <= 3 tiles) of one 64 x 64 quadrant are
// staged in shared memory, two quadrants in flight (reusing the ring after the main loop)
constexpr int k2QLD = 64 + 4;
constexpr int k2QOpFloats = 64 * k2QLD;
constexpr int k2QBufFloats = 3 * k2QOpFloats;
constexpr int k2EpiFloats = 2 * k2QBufFloats;  // 102 KB
constexpr int k2MaxFloats = k2RingFloats > k2EpiFloats ? k2RingFloats : k2EpiFloats;
constexpr int k2SmemFloats = k2MaxFloats > kPairFloats ? k2MaxFloats : kPairFloats;
constexpr int k2SmemBytes = k2SmemFloats * 4;
static_assert(CNP2_CTAS * (k2SmemBytes + 1024) <= 228 * 1024, "CTAs per SM");

template <int TILE>
struct GraphCfg;
template <>
struct GraphCfg<64> {
  static constexpr int threads = kThreads, ctas_per_sm = 1, smem = kSmemBytes;
};
template <>
struct GraphCfg<128> {
  static constexpr int threads = k2Threads, ctas_per_sm = CNP2_CTAS, smem = k2SmemBytes;
};

__device__ __forceinline__ void cp_async16(float* smem_dst, const float* gsrc) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ float4 ldcg4(const float* p) {
  return __ldcg(reinterpret_cast<const float4*>(p));
}
__device__ __forceinline__ void st4(float* p, float a, float b, float c, float d) {
  __stcg(reinterpret_cast<float4*>(p), make_float4(a, b, c, d));
}
__device__ __forceinline__ unsigned short bf16_bits(float x) {
  const __nv_bfloat16 h = __float2bfloat16_rn(x);
  return *reinterpret_cast<const unsigned short*>(&h);
}
__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ unsigned long long gtimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void tile_pair(int nt, int t, int& I, int& J) {
  I = 0;
  while (t >= nt - I) {
    t -= nt - I;
    ++I;
  }
  J = I + t;
}

__device__ __forceinline__ int64_t tri_idx(int i, int j, int b) {
  return (int64_t)i * b - (int64_t)i * (i + 1) / 2 + (j - i - 1);
}

#if CNP2_FMA2
// Product k steps on packed pairs: fma.rn.f32x2 does two independent fp32 fused
// multiply-adds (each rounded once, as fmaf), so an outer-product step of 2P x 2Q
// accumulators takes 2PQ issue slots instead of 4PQ, in the same per-element order over k.
// Accumulator pairs:
//   D[p][q] = (acc[2p][2q],     acc[2p + 1][2q + 1]) += (a[2p], a[2p + 1]) * (b[2q], b[2q + 1])
//   X[p][q] = (acc[2p][2q + 1], acc[2p + 1][2q])     += (a[2p], a[2p + 1]) * (b[2q + 1], b[2q])
// so the a and b pairs are halves of 16-byte shared-memory loads; only the swapped b pairs
// are built per k step.
__device__ __forceinline__ void fma2(unsigned long long& d, unsigned long long a,
                                     unsigned long long b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(d) : "l"(a), "l"(b));
}
__device__ __forceinline__ unsigned long long swap_pair(unsigned long long v) {
  unsigned long long r;
  asm("{\n\t.reg .b32 lo, hi;\n\tmov.b64 {lo, hi}, %1;\n\tmov.b64 %0, {hi, lo};\n\t}"
      : "=l"(r) : "l"(v));
  return r;
}
template <int NP, int NQ>
__device__ __forceinline__ void outer2(unsigned long long (&D)[NP][NQ],
                                       unsigned long long (&X)[NP][NQ],
                                       const unsigned long long (&a)[NP],
                                       const unsigned long long (&b)[NQ]) {
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    const unsigned long long bs = swap_pair(b[q]);
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      fma2(D[p][q], a[p], b[q]);
      fma2(X[p][q], a[p], bs);
    }
  }
}
template <int NP, int NQ>
__device__ __forceinline__ void zero2(unsigned long long (&D)[NP][NQ],
                                      unsigned long long (&X)[NP][NQ]) {
#pragma unroll
  for (int p = 0; p < NP; ++p)
#pragma unroll
    for (int q = 0; q < NQ; ++q) D[p][q] = X[p][q] = 0ull;  // (+0.f, +0.f)
}
template <int NP, int NQ>
__device__ __forceinline__ void scale2(unsigned long long (&D)[NP][NQ],
                                       unsigned long long (&X)[NP][NQ], float f) {
  unsigned long long ff;
  asm("mov.b64 %0, {%1, %1};" : "=l"(ff) : "f"(f));
#pragma unroll
  for (int p = 0; p < NP; ++p)
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      asm("mul.rn.f32x2 %0, %0, %1;" : "+l"(D[p][q]) : "l"(ff));
      asm("mul.rn.f32x2 %0, %0, %1;" : "+l"(X[p][q]) : "l"(ff));
    }
}
template <int NP, int NQ>
__device__ __forceinline__ void unpack2(const unsigned long long (&D)[NP][NQ],
                                        const unsigned long long (&X)[NP][NQ],
                                        float (&acc)[2 * NP][2 * NQ]) {
#pragma unroll
  for (int p = 0; p < NP; ++p)
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      asm("mov.b64 {%0, %1}, %2;" : "=f"(acc[2 * p][2 * q]), "=f"(acc[2 * p + 1][2 * q + 1])
          : "l"(D[p][q]));
      asm("mov.b64 {%0, %1}, %2;" : "=f"(acc[2 * p][2 * q + 1]), "=f"(acc[2 * p + 1][2 * q])
          : "l"(X[p][q]));
    }
}
#endif

// ------------------------------------------------------------------ product tile
// C-tile (64 x 64) of one block: acc = op(A1) B1 (+ alpha2 op(A2) B2), every A read by rows
// (symmetric, skew, or given transposed), then the structured epilogue.
__device__ void product_tile64(const CnpJob& J, int z, int t, int b, float* smem) {
  const int tid = threadIdx.x;
  const int grp = tid >> 7, gtid = tid & (kGThreads - 1);
  const int tx = gtid & 15, ty = gtid >> 4;
  const int nt = b / 64;
  int I, Jt;
  if (J.mode == SG_FULL) {
    I = t / nt;
    Jt = t - I * nt;
  } else {
    tile_pair(nt, t, I, Jt);
  }
  const int m0 = I * 64, n0 = Jt * 64;
  const int64_t boff = (int64_t)z * b * b;
  const float* A1 = J.A + boff;
  const float* B1 = J.B + boff;
  const float* A2 = J.A2 ? J.A2 + boff : nullptr;
  const float* B2 = J.B2 ? J.B2 + boff : nullptr;
  const int nk1 = b / kBK;
  const int nk2 = A2 ? b / kBK : 0;
  const int nkt = nk1 + nk2;
  // this group's k tiles
  const int kt_begin = (grp * nkt) / kGroups;
  const int kt_end = ((grp + 1) * nkt) / kGroups;
  const float s1 = J.a_sym < 0 ? -1.f : 1.f;
  const float s2 = J.a2_sym < 0 ? -1.f : 1.f;
  const float boundary = s1 * s2 * J.alpha2;
  // the group's accumulators times g_scale are its share of op(A1)B1 + alpha2 op(A2)B2
  const float g_scale = (nk2 > 0 && kt_end > nk1) ? s2 * J.alpha2 : s1;

  float acc[8][4];
#if CNP2_FMA2
  unsigned long long accD[4][2], accX[4][2];
  zero2(accD, accX);
#else
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;
#endif

  float* ring = smem + grp * kStages * kStageFloats;
  auto As_ = [&](int st) { return reinterpret_cast<float (*)[kLD]>(ring + st * kStageFloats); };
  auto Bs_ = [&](int st) {
    return reinterpret_cast<float (*)[kLD]>(ring + st * kStageFloats + kBK * kLD);
  };
  auto issue = [&](int kt) {  // kt: absolute k tile index
    if (kt < kt_end) {
      const bool first = kt < nk1;
      const float* A = first ? A1 : A2;
      const float* B = first ? B1 : B2;
      const int k0 = (first ? kt : kt - nk1) * kBK;
      const int st = (kt - kt_begin) % kStages;
      float (*As)[kLD] = As_(st);
      float (*Bs)[kLD] = Bs_(st);
#pragma unroll
      for (int l = 0; l < 2; ++l) {
        const int f = gtid + l * kGThreads;
        const int r = f >> 4, c4 = (f & 15) * 4;
        cp_async16(&As[r][c4], A + (int64_t)(k0 + r) * b + m0 + c4);
        cp_async16(&Bs[r][c4], B + (int64_t)(k0 + r) * b + n0 + c4);
      }
    }
    cp_commit();
  };
  // named barrier per group (ids 1..4; 0 is __syncthreads)
  auto group_sync = [&]() {
    asm volatile("bar.sync %0, %1;" ::"r"(grp + 1), "r"(kGThreads) : "memory");
  };
#pragma unroll
  for (int st = 0; st < kStages - 1; ++st) issue(kt_begin + st);
  // epilogue operand tiles: one cp.async group of their own, committed after the first
  // kStages - 1 k tiles, so they queue behind the operands the mainloop needs first
  {
    float* E = smem + kRingFloats;
    auto fetch = [&](int e, const float* src, int row0, int col0) {
      const float* g0 = src + boff + (int64_t)row0 * b + col0;
#pragma unroll
      for (int l = 0; l < 64 * 16 / kThreads; ++l) {
        const int f = tid + l * kThreads;
        const int r = f >> 4, c4 = (f & 15) * 4;
        cp_async16(E + e * 64 * kELD + r * kELD + c4, g0 + (int64_t)r * b + c4);
      }
    };
    for (int q = 0; q < J.nadd; ++q) fetch(q, J.add[q], m0, n0);
    if (J.skew_add) fetch(J.nadd, J.skew_add, m0, n0);
    cp_commit();
  }
  for (int kt = kt_begin; kt < kt_end; ++kt) {
    // k tile kt is complete once at most kStages - 2 later groups are pending (plus the
    // epilogue group while it is still younger than kt)
    if (kt - kt_begin < kStages - 1) cp_wait<kStages - 1>(); else cp_wait<kStages - 2>();
    group_sync();
    issue(kt + kStages - 1);
    const int st = (kt - kt_begin) % kStages;
    float (*As)[kLD] = As_(st);
    float (*Bs)[kLD] = Bs_(st);
#if CNP2_FMA2
    if (nk2 > 0 && kt == nk1 && kt > kt_begin) scale2(accD, accX, boundary);
#pragma unroll
    for (int k = 0; k < kBK; ++k) {
      const ulonglong2 a0 = *reinterpret_cast<const ulonglong2*>(&As[k][ty * 8]);
      const ulonglong2 a1 = *reinterpret_cast<const ulonglong2*>(&As[k][ty * 8 + 4]);
      const ulonglong2 bv = *reinterpret_cast<const ulonglong2*>(&Bs[k][tx * 4]);
      const unsigned long long a[4] = {a0.x, a0.y, a1.x, a1.y};
      const unsigned long long bb[2] = {bv.x, bv.y};
      outer2(accD, accX, a, bb);
    }
#else
    if (nk2 > 0 && kt == nk1 && kt > kt_begin) {
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] *= boundary;
    }
#pragma unroll
    for (int k = 0; k < kBK; ++k) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[k][ty * 8]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[k][ty * 8 + 4]);
      const float4 bv = *reinterpret_cast<const float4*>(&Bs[k][tx * 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bb[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(a[r], bb[c], acc[r][c]);
    }
#endif
  }
#if CNP2_FMA2
  unpack2(accD, accX, acc);
#endif
  cp_wait<0>();
  __syncthreads();  // every group is done with its ring: the space becomes red[]

  // partial tiles -> red[grp][row][col]
  float* red = smem;
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    float* dst = red + (grp * 64 + ty * 8 + r) * 64 + tx * 4;
    *reinterpret_cast<float4*>(dst) = make_float4(g_scale * acc[r][0], g_scale * acc[r][1],
                                                  g_scale * acc[r][2], g_scale * acc[r][3]);
  }
  __syncthreads();
  // epilogue: thread owns row il and 8 consecutive columns of the tile
  // sym = diag*delta + sum addc*add;  skew = alpha*acc + skew_c*skew_add
  // The job's scalars are read into registers before the first store, and every store is
  // an explicit global-space store, so no store can be taken to overwrite shared memory.
  float* const C = J.C + boff;
  __nv_bfloat16* const Cb = J.Cb ? J.Cb + boff : nullptr;
  float* const C2 = J.C2 ? J.C2 + boff : nullptr;
  const int mode = J.mode;
  const bool structured = mode != SG_FULL;
  const float alpha = J.alpha, diag = J.diag, diag2 = J.diag2, alpha_c2 = J.alpha_c2;
  const float skew_c = J.skew_c;
  const int nadd = J.nadd;
  const bool has_skew = J.skew_add != nullptr;
  float addc[kEpiTiles], addc2[kEpiTiles];
#pragma unroll
  for (int q = 0; q < kEpiTiles; ++q) {
    addc[q] = q < nadd ? J.addc[q] : 0.f;
    addc2[q] = q < nadd ? J.addc2[q] : 0.f;
  }
  float (*Ms)[65] = reinterpret_cast<float (*)[65]>(smem + kRedFloats);
  float (*Ms2)[65] = reinterpret_cast<float (*)[65]>(smem + kRedFloats + 64 * 65);
#pragma unroll 1
  for (int pass = 0; pass < 64 * 64 / (8 * kThreads); ++pass) {
    const int il = pass * (kThreads / 8) + (tid >> 3), jl0 = (tid & 7) * 8;
    const int i = m0 + il, j0 = n0 + jl0;
    const int64_t row = (int64_t)i * b;
    float a[8];
    {
      const float* r0 = red + il * 64 + jl0;
      const float4 p0 = *reinterpret_cast<const float4*>(r0);
      const float4 p1 = *reinterpret_cast<const float4*>(r0 + 4);
      a[0] = p0.x; a[1] = p0.y; a[2] = p0.z; a[3] = p0.w;
      a[4] = p1.x; a[5] = p1.y; a[6] = p1.z; a[7] = p1.w;
#pragma unroll
      for (int g2 = 1; g2 < kGroups; ++g2) {  // fixed summation order
        const float* rg = r0 + g2 * 64 * 64;
        const float4 q0 = *reinterpret_cast<const float4*>(rg);
        const float4 q1 = *reinterpret_cast<const float4*>(rg + 4);
        a[0] += q0.x; a[1] += q0.y; a[2] += q0.z; a[3] += q0.w;
        a[4] += q1.x; a[5] += q1.y; a[6] += q1.z; a[7] += q1.w;
      }
    }
    float sym[8], sym2[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const bool dg = (i == j0 + c);
      sym[c] = dg ? diag : 0.f;
      sym2[c] = dg ? diag2 : 0.f;
    }
    const float* E = smem + kRingFloats + il * kELD + jl0;
#pragma unroll
    for (int q = 0; q < kEpiTiles; ++q) {
      if (q >= nadd) break;
      const float4 x0 = *reinterpret_cast<const float4*>(E + q * 64 * kELD);
      const float4 x1 = *reinterpret_cast<const float4*>(E + q * 64 * kELD + 4);
      const float xs[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        sym[c] += addc[q] * xs[c];
        sym2[c] += addc2[q] * xs[c];
      }
    }
    float skew[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) skew[c] = alpha * a[c];
    if (has_skew) {
      const float4 x0 = *reinterpret_cast<const float4*>(E + nadd * 64 * kELD);
      const float4 x1 = *reinterpret_cast<const float4*>(E + nadd * 64 * kELD + 4);
      const float xs[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
      for (int c = 0; c < 8; ++c) skew[c] += skew_c * xs[c];
    }
    float v[8], vm[8], v2[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int j = j0 + c;
      if (mode == SG_SYMSKEW) {
        v[c] = (i == j) ? sym[c] : sym[c] + skew[c];
        vm[c] = sym[c] - skew[c];
      } else {
        v[c] = skew[c] + sym[c];
        vm[c] = v[c];
      }
      v2[c] = alpha_c2 * a[c] + sym2[c];
    }
    if (structured) {  // mirror staging first: shared-memory work before the stores
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        Ms[il][jl0 + c] = vm[c];
        if (C2) Ms2[il][jl0 + c] = v2[c];
      }
    }
    if (structured && I == Jt) {  // diagonal tile: this thread writes the upper triangle only
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int j = j0 + c;
        if (i <= j) {
          __stcg(C + row + j, v[c]);
          if (Cb) __stcg(reinterpret_cast<unsigned short*>(Cb + row + j), bf16_bits(v[c]));
          if (C2) __stcg(C2 + row + j, v2[c]);
        }
      }
    } else {
      __stcg(reinterpret_cast<float4*>(C + row + j0), make_float4(v[0], v[1], v[2], v[3]));
      __stcg(reinterpret_cast<float4*>(C + row + j0 + 4), make_float4(v[4], v[5], v[6], v[7]));
      if (Cb) {
        const uint4 o = make_uint4(bf16x2_bits(v[0], v[1]), bf16x2_bits(v[2], v[3]),
                                   bf16x2_bits(v[4], v[5]), bf16x2_bits(v[6], v[7]));
        __stcg(reinterpret_cast<uint4*>(Cb + row + j0), o);
      }
      if (C2) {
        __stcg(reinterpret_cast<float4*>(C2 + row + j0), make_float4(v2[0], v2[1], v2[2], v2[3]));
        __stcg(reinterpret_cast<float4*>(C2 + row + j0 + 4),
               make_float4(v2[4], v2[5], v2[6], v2[7]));
      }
    }
  }  // passes
  if (structured) {
    __syncthreads();  // staged mirror values of every pass are visible
    // row jl of the mirrored tile is column jl of this one; a thread writes 4 consecutive
    // elements (wide stores: the store count, not the bytes, sets the cost here)
#pragma unroll 1
    for (int e = tid; e < 64 * 16; e += kThreads) {
      const int jl = e >> 4, il4 = (e & 15) * 4;
      const int64_t ji = (int64_t)(n0 + jl) * b + m0 + il4;
      const float4 v = make_float4(Ms[il4][jl], Ms[il4 + 1][jl], Ms[il4 + 2][jl], Ms[il4 + 3][jl]);
      float4 v2 = make_float4(0.f, 0.f, 0.f, 0.f);
      if (C2) v2 = make_float4(Ms2[il4][jl], Ms2[il4 + 1][jl], Ms2[il4 + 2][jl], Ms2[il4 + 3][jl]);
      if (I != Jt) {
        __stcg(reinterpret_cast<float4*>(C + ji), v);
        if (Cb)
          __stcg(reinterpret_cast<uint2*>(Cb + ji),
                 make_uint2(bf16x2_bits(v.x, v.y), bf16x2_bits(v.z, v.w)));
        if (C2) __stcg(reinterpret_cast<float4*>(C2 + ji), v2);
      } else {  // diagonal tile: the strictly lower triangle only
        const float vv[4] = {v.x, v.y, v.z, v.w};
        const float ww[4] = {v2.x, v2.y, v2.z, v2.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (il4 + u >= jl) continue;
          __stcg(C + ji + u, vv[u]);
          if (Cb) __stcg(reinterpret_cast<unsigned short*>(Cb + ji + u), bf16_bits(vv[u]));
          if (C2) __stcg(C2 + ji + u, ww[u]);
        }
      }
    }
  }
}

// ------------------------------------------------------------------ 128 x 128 product tile
// The same product and epilogue as product_tile64 on a 128 x 128 output tile, for 256
// threads: thread (tx, ty) = (tid & 15, tid >> 4) owns rows {4 ty .. 4 ty + 3} and
// {64 + 4 ty .. 64 + 4 ty + 3} and the same two column quads from 4 tx, so each k step
// reads four 16-byte shared-memory vectors (conflict-free: a quarter warp reads 128
// contiguous bytes or one broadcast address) for 64 FMAs.  The whole K runs in one
// thread (no split, no partial-tile reduction); the epilogue works quadrant by quadrant
// from the accumulator registers: operand rows are read as 16-byte vectors, the tile is
// stored with 16-byte row stores, and the mirror of a symmetric (or symmetric + skew)
// result is transposed through shared memory and stored as whole rows too.
// One k slice of the 128 x 128 item: acc[r][c] += A[k][row r] B[k][col c] for the thread's
// rows {4 ty + r} U {64 + 4 ty + r} and columns {4 tx + c} U {64 + 4 tx + c}.
__device__ __forceinline__ void kslice128(float (&acc)[8][8], const float* As, const float* Bs,
                                          int tx, int ty) {
#pragma unroll k2KUnroll
  for (int k = 0; k < k2BK; ++k) {
    const float4 a0 = *reinterpret_cast<const float4*>(As + k * k2LD + ty * 4);
    const float4 a1 = *reinterpret_cast<const float4*>(As + k * k2LD + 64 + ty * 4);
    const float4 b0 = *reinterpret_cast<const float4*>(Bs + k * k2LD + tx * 4);
    const float4 b1 = *reinterpret_cast<const float4*>(Bs + k * k2LD + 64 + tx * 4);
    const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[r][c] = fmaf(a[r], bb[c], acc[r][c]);
  }
}


#if CNP2_FMA2
// One k slice of the 128 x 128 item on packed pairs.  LOWER_LEFT = false skips the
// quadrant below the diagonal (rows 64.., columns ..63: pairs p >= 2, q < 2) of a diagonal
// tile of a symmetric result, which the epilogue never stores.
template <bool LOWER_LEFT>
__device__ __forceinline__ void kslice128_x2(unsigned long long (&D)[4][4],
                                             unsigned long long (&X)[4][4], const float* As,
                                             const float* Bs, int tx, int ty) {
#pragma unroll k2KUnroll
  for (int k = 0; k < k2BK; ++k) {
    const ulonglong2 a0 = *reinterpret_cast<const ulonglong2*>(As + k * k2LD + ty * 4);
    const ulonglong2 a1 = *reinterpret_cast<const ulonglong2*>(As + k * k2LD + 64 + ty * 4);
    const ulonglong2 b0 = *reinterpret_cast<const ulonglong2*>(Bs + k * k2LD + tx * 4);
    const ulonglong2 b1 = *reinterpret_cast<const ulonglong2*>(Bs + k * k2LD + 64 + tx * 4);
    const unsigned long long a[4] = {a0.x, a0.y, a1.x, a1.y};
    const unsigned long long bb[4] = {b0.x, b0.y, b1.x, b1.y};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const unsigned long long bs = swap_pair(bb[q]);
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        if (!LOWER_LEFT && p >= 2 && q < 2) continue;
        fma2(D[p][q], a[p], bb[q]);
        fma2(X[p][q], a[p], bs);
      }
    }
  }
}
#endif

__device__ void product_tile128(const CnpJob& J, int z, int t, int b, float* smem) {
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int nt = b / 128;
  int I, Jt;
  if (J.mode == SG_FULL) {
    I = t / nt;
    Jt = t - I * nt;
  } else {
    tile_pair(nt, t, I, Jt);
  }
  const int m0 = I * 128, n0 = Jt * 128;
  // a diagonal tile of a symmetric (or symmetric + skew) result stores only i <= j
  const bool skip_ll = J.mode != SG_FULL && I == Jt;
  const int64_t boff = (int64_t)z * b * b;
  const float* A1 = J.A + boff;
  const float* B1 = J.B + boff;
  const float* A2 = J.A2 ? J.A2 + boff : nullptr;
  const float* B2 = J.B2 ? J.B2 + boff : nullptr;
  const int nk1 = b / k2BK;
  const int nkt = nk1 + (A2 ? b / k2BK : 0);
  const float s1 = J.a_sym < 0 ? -1.f : 1.f;
  const float s2 = J.a2_sym < 0 ? -1.f : 1.f;
  // raw sums run over A read by rows; the first part is rescaled at the boundary so that
  // one final factor gives op(A1) B1 + alpha2 op(A2) B2 (alpha2 = +-1 in every job)
  const float boundary = s1 * s2 * J.alpha2;
  const float scale = A2 ? s2 * J.alpha2 : s1;

  float acc[8][8];
#if CNP2_FMA2
  unsigned long long accD[4][4], accX[4][4];
  zero2(accD, accX);
#else
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[r][c] = 0.f;
#endif

  auto As_ = [&](int st) { return smem + st * k2StageFloats; };
  auto Bs_ = [&](int st) { return smem + st * k2StageFloats + k2BK * k2LD; };
  auto issue = [&](int kt) {
    if (kt < nkt) {
      const bool first = kt < nk1;
      const float* A = first ? A1 : A2;
      const float* B = first ? B1 : B2;
      const int k0 = (first ? kt : kt - nk1) * k2BK;
      float* As = As_(kt % k2Stages);
      float* Bs = Bs_(kt % k2Stages);
#pragma unroll
      for (int l = 0; l < k2BK * 32 / k2Threads; ++l) {
        const int f = tid + l * k2Threads;
        const int r = f >> 5, c4 = (f & 31) * 4;
        cp_async16(As + r * k2LD + c4, A + (int64_t)(k0 + r) * b + m0 + c4);
        cp_async16(Bs + r * k2LD + c4, B + (int64_t)(k0 + r) * b + n0 + c4);
      }
    }
    cp_commit();
  };
#pragma unroll
  for (int st = 0; st < k2Stages - 1; ++st) issue(st);
  for (int kt = 0; kt < nkt; ++kt) {
    cp_wait<k2Stages - 2>();
    __syncthreads();  // k tile kt landed for every thread; tile kt - 1 fully consumed
    issue(kt + k2Stages - 1);
    const float* As = As_(kt % k2Stages);
    const float* Bs = Bs_(kt % k2Stages);
#if CNP2_FMA2
    if (kt == nk1) scale2(accD, accX, boundary);  // only with a second product
    if (CNP2_DIAGSKIP && skip_ll)
      kslice128_x2<false>(accD, accX, As, Bs, tx, ty);
    else
      kslice128_x2<true>(accD, accX, As, Bs, tx, ty);
#else
    if (kt == nk1) {  // only with a second product
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[r][c] *= boundary;
    }
#if CNP2_DBUF
    float4 a0 = *reinterpret_cast<const float4*>(As + ty * 4);
    float4 a1 = *reinterpret_cast<const float4*>(As + 64 + ty * 4);
    float4 b0 = *reinterpret_cast<const float4*>(Bs + tx * 4);
    float4 b1 = *reinterpret_cast<const float4*>(Bs + 64 + tx * 4);
#pragma unroll k2KUnroll
    for (int k = 0; k < k2BK; ++k) {
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
      if (k + 1 < k2BK) {  // the next k step's fragments load while this one computes
        a0 = *reinterpret_cast<const float4*>(As + (k + 1) * k2LD + ty * 4);
        a1 = *reinterpret_cast<const float4*>(As + (k + 1) * k2LD + 64 + ty * 4);
        b0 = *reinterpret_cast<const float4*>(Bs + (k + 1) * k2LD + tx * 4);
        b1 = *reinterpret_cast<const float4*>(Bs + (k + 1) * k2LD + 64 + tx * 4);
      }
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[r][c] = fmaf(a[r], bb[c], acc[r][c]);
    }
#else
    kslice128(acc, As, Bs, tx, ty);
#endif
#endif
  }
  cp_wait<0>();
#if CNP2_FMA2
  unpack2(accD, accX, acc);
#endif

  // ---- epilogue from the registers, quadrant by quadrant
  // sym = diag*delta + sum addc*add;  skew = alpha*acc + skew_c*skew_add
  float* const C = J.C + boff;
  __nv_bfloat16* const Cb = J.Cb ? J.Cb + boff : nullptr;
  float* const C2 = J.C2 ? J.C2 + boff : nullptr;
  const int mode = J.mode;
  const bool structured = mode != SG_FULL;
  const float alpha = J.alpha * scale, alpha_c2 = J.alpha_c2 * scale;
  const float diag = J.diag, diag2 = J.diag2, skew_c = J.skew_c;
  const int nadd = J.nadd;
  const float* ops[3] = {nadd > 0 ? J.add[0] + boff : nullptr,
                         nadd > 1 ? J.add[1] + boff : nullptr,
                         J.skew_add ? J.skew_add + boff : nullptr};
  const float ac0 = nadd > 0 ? J.addc[0] : 0.f, ac1 = nadd > 1 ? J.addc[1] : 0.f;
  const float bc0 = nadd > 0 ? J.addc2[0] : 0.f, bc1 = nadd > 1 ? J.addc2[1] : 0.f;
  const bool has_ops = nadd > 0 || J.skew_add;
  const bool diag_tile = structured && I == Jt;
  // quadrants that produce output (q = 2 qr + qc): a diagonal tile keeps i <= j, so its
  // quadrant below the diagonal (q = 2: rows 64.., columns ..63) holds nothing to store
  const int nq = diag_tile ? 3 : 4;
  auto quad = [&](int qi) { return (diag_tile && qi == 2) ? 3 : qi; };
  // the ring is free: every thread passed the last k tile's barrier and its loads landed
  __syncthreads();
  auto stage_ops = [&](int qi) {  // coalesced 16-byte copies of the quadrant's operands
    if (has_ops && qi < nq) {
      const int qr = quad(qi) >> 1, qc = quad(qi) & 1;
      float* buf = smem + (qi & 1) * k2QBufFloats;
#pragma unroll
      for (int o = 0; o < 3; ++o) {
        if (!ops[o]) continue;
        const float* src = ops[o] + (int64_t)(m0 + qr * 64) * b + n0 + qc * 64;
#pragma unroll
        for (int l = 0; l < 4; ++l) {
          const int f = tid + l * k2Threads;
          const int r = f >> 4, c4 = (f & 15) * 4;
          cp_async16(buf + o * k2QOpFloats + r * k2QLD + c4, src + (int64_t)r * b + c4);
        }
      }
    }
    cp_commit();
  };
  stage_ops(0);
  stage_ops(1);
  // the quadrant loop is unrolled so that the accumulators are indexed by constants
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    if (diag_tile && q == 2) continue;
    const int qi = (diag_tile && q == 3) ? 2 : q;  // position in the staging order
    cp_wait<1>();
    __syncthreads();  // quadrant qi's operands are in shared memory for every thread
    const int qr = q >> 1, qc = q & 1;
    const bool dq = diag_tile && qr == qc;  // element-wise i <= j / i < j masks
    const int i0 = m0 + qr * 64 + ty * 4, j0 = n0 + qc * 64 + tx * 4;
    const float* buf = smem + (qi & 1) * k2QBufFloats;
    // Row rr of the thread's 4 x 4 piece: its staged operands (one 16-byte load per operand),
    // the direct values v (at (i, j)), the mirrored values vm (at (j, i)) and the second
    // output v2, all from registers; vm and v2 are kept for the mirror's column stores.
    float vmq[4][4], v2q[4][4];
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int i = i0 + rr;
      const int so = (ty * 4 + rr) * k2QLD + tx * 4;
      const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 e0v = ops[0] ? *reinterpret_cast<const float4*>(buf + so) : z4;
      const float4 e1v = ops[1] ? *reinterpret_cast<const float4*>(buf + k2QOpFloats + so) : z4;
      const float4 esv = ops[2] ? *reinterpret_cast<const float4*>(buf + 2 * k2QOpFloats + so) : z4;
      const float e0[4] = {e0v.x, e0v.y, e0v.z, e0v.w};
      const float e1[4] = {e1v.x, e1v.y, e1v.z, e1v.w};
      const float es[4] = {esv.x, esv.y, esv.z, esv.w};
      float v[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int j = j0 + c;
        const float a = acc[qr * 4 + rr][qc * 4 + c];
        const float sym = (i == j ? diag : 0.f) + ac0 * e0[c] + ac1 * e1[c];
        const float sym2 = (i == j ? diag2 : 0.f) + bc0 * e0[c] + bc1 * e1[c];
        const float skew = alpha * a + skew_c * es[c];
        if (mode == SG_SYMSKEW) {
          v[c] = (i == j) ? sym : sym + skew;
          vmq[rr][c] = sym - skew;
        } else {
          v[c] = skew + sym;
          vmq[rr][c] = v[c];
        }
        v2q[rr][c] = alpha_c2 * a + sym2;
      }
      // direct: row i, columns j0 .. j0 + 3
      const int64_t row = (int64_t)i * b;
      if (!dq) {
        __stcg(reinterpret_cast<float4*>(C + row + j0), make_float4(v[0], v[1], v[2], v[3]));
        if (Cb)
          __stcg(reinterpret_cast<uint2*>(Cb + row + j0),
                 make_uint2(bf16x2_bits(v[0], v[1]), bf16x2_bits(v[2], v[3])));
        if (C2)
          __stcg(reinterpret_cast<float4*>(C2 + row + j0),
                 make_float4(v2q[rr][0], v2q[rr][1], v2q[rr][2], v2q[rr][3]));
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (i > j0 + c) continue;
          __stcg(C + row + j0 + c, v[c]);
          if (Cb) __stcg(reinterpret_cast<unsigned short*>(Cb + row + j0 + c), bf16_bits(v[c]));
          if (C2) __stcg(C2 + row + j0 + c, v2q[rr][c]);
        }
      }
    }
    if (structured) {
      // mirror: element (i, j) of the quadrant goes to (j, i).  The thread's 4 x 4 pieces of
      // the mirrored values are transposed through the quadrant's staging buffer (its
      // operands are in registers by now), so that the mirror is stored as whole rows.
      __syncthreads();  // every thread has read its operands from buffer (qi & 1)
      float* tb = smem + (qi & 1) * k2QBufFloats;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        *reinterpret_cast<float4*>(tb + (tx * 4 + c) * k2QLD + ty * 4) =
            make_float4(vmq[0][c], vmq[1][c], vmq[2][c], vmq[3][c]);
        if (C2)
          *reinterpret_cast<float4*>(tb + k2QOpFloats + (tx * 4 + c) * k2QLD + ty * 4) =
              make_float4(v2q[0][c], v2q[1][c], v2q[2][c], v2q[3][c]);
      }
      __syncthreads();
      // mirrored quadrant: rows n0 + qc 64 .., columns m0 + qr 64 ..; a warp stores two
      // contiguous 256-byte row segments per instruction
#pragma unroll
      for (int l = 0; l < 4; ++l) {
        const int f = tid + l * k2Threads;
        const int r = f >> 4, c4 = (f & 15) * 4;
        const int jg = n0 + qc * 64 + r, ig = m0 + qr * 64 + c4;
        const float4 w = *reinterpret_cast<const float4*>(tb + r * k2QLD + c4);
        const float4 w2 = C2 ? *reinterpret_cast<const float4*>(tb + k2QOpFloats + r * k2QLD + c4)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
        const int64_t row = (int64_t)jg * b;
        if (!dq) {
          __stcg(reinterpret_cast<float4*>(C + row + ig), w);
          if (Cb)
            __stcg(reinterpret_cast<uint2*>(Cb + row + ig),
                   make_uint2(bf16x2_bits(w.x, w.y), bf16x2_bits(w.z, w.w)));
          if (C2) __stcg(reinterpret_cast<float4*>(C2 + row + ig), w2);
        } else {  // strictly below the diagonal only: (j, i) with i < j
          const float wv[4] = {w.x, w.y, w.z, w.w};
          const float w2v[4] = {w2.x, w2.y, w2.z, w2.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (ig + e >= jg) continue;
            __stcg(C + row + ig + e, wv[e]);
            if (Cb) __stcg(reinterpret_cast<unsigned short*>(Cb + row + ig + e), bf16_bits(wv[e]));
            if (C2) __stcg(C2 + row + ig + e, w2v[e]);
          }
        }
      }
    }
    __syncthreads();  // every thread is done with buffer (qi & 1) before it is refilled
    stage_ops(qi + 2);
  }
  cp_wait<0>();
}

// ------------------------------------------------------------------ 64 x 64 tile-pair jobs
// Tile pair (I, J), I <= J, of a block; thread (tx = tid & 63, ty = tid >> 6) walks rows
// ty, ty + 8, ... of the 64 x 64 tile, so each row is one coalesced 256-byte access.

// With NT threads, a thread handles 4 consecutive columns c4.. of rows
// r = (tid >> 4) + (NT / 16) u of a tile: every global access is a 16-byte vector of a
// coalesced row (the number of requests, not the bytes, bounds these small jobs), and all
// of a thread's loads are issued before any of them is used, so a tile costs one L2 round
// trip.


// theta -> Q: Q_ij = theta, Q_ji = -theta
template <int NT>
__device__ void expand_tile(const CnpJob& J, int z, int t, int b, float* smem) {
  constexpr int kQuadRows = NT / 16, kQuadSweeps = kPT / kQuadRows;
  static_assert(kQuadRows * kQuadSweeps == kPT, "tile sweep");
  float (*tt)[kPLD] = reinterpret_cast<float (*)[kPLD]>(smem);
  int I, Jt;
  tile_pair(b / kPT, t, I, Jt);
  const int64_t ntri = (int64_t)b * (b - 1) / 2;
  const float* th = J.A + z * ntri;
  float* q = J.C + (int64_t)z * b * b;
  const int c4 = (threadIdx.x & 15) * 4, r0 = threadIdx.x >> 4;
  float v[kQuadSweeps][4];
#pragma unroll
  for (int u = 0; u < kQuadSweeps; ++u) {
    const int i = I * kPT + r0 + u * kQuadRows;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int j = Jt * kPT + c4 + w;
      v[u][w] = (i < j) ? __ldcg(th + tri_idx(i, j, b)) : 0.f;
    }
  }
#pragma unroll
  for (int u = 0; u < kQuadSweeps; ++u)
#pragma unroll
    for (int w = 0; w < 4; ++w) tt[r0 + u * kQuadRows][c4 + w] = v[u][w];
  __syncthreads();
#pragma unroll
  for (int u = 0; u < kQuadSweeps; ++u) {
    const int r = r0 + u * kQuadRows;
    float o[4], m[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int c = c4 + w;
      o[w] = (I == Jt && r > c) ? -tt[c][r] : tt[r][c];
      m[w] = -tt[c][r];
    }
    st4(q + (int64_t)(I * kPT + r) * b + Jt * kPT + c4, o[0], o[1], o[2], o[3]);
    if (I != Jt) st4(q + (int64_t)(Jt * kPT + r) * b + I * kPT + c4, m[0], m[1], m[2], m[3]);
  }
}

// out_o = sum_s coef[o][s] (X_s + X_s^T) (symmetric outputs), optional Cb_f = X_0^T.
// Both tiles (I,J) and (J,I) of every input are staged first; each output element is then
// formed directly (the sum is commutative, so diagonal tiles come out exactly symmetric).
template <int NT>
__device__ void symcomb_tile(const CnpJob& J, int z, int t, int b, float* smem) {
  constexpr int kQuadRows = NT / 16, kQuadSweeps = kPT / kQuadRows;
  static_assert(kQuadRows * kQuadSweeps == kPT, "tile sweep");
  float (*ta)[kPT][kPLD] = reinterpret_cast<float (*)[kPT][kPLD]>(smem);            // X_s(I,J)
  float (*tb)[kPT][kPLD] = reinterpret_cast<float (*)[kPT][kPLD]>(smem + 2 * kPT * kPLD);  // X_s(J,I)
  int I, Jt;
  tile_pair(b / kPT, t, I, Jt);
  const int64_t base = (int64_t)z * b * b;
  const int c4 = (threadIdx.x & 15) * 4, r0 = threadIdx.x >> 4;
  const int nin = J.nin, nout = J.nout;
  float4 va[2][kQuadSweeps], vb[2][kQuadSweeps];
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    if (s >= nin) break;
    const float* x = (s == 0 ? J.A : J.B) + base;
#pragma unroll
    for (int u = 0; u < kQuadSweeps; ++u) {
      const int r = r0 + u * kQuadRows;
      va[s][u] = ldcg4(x + (int64_t)(I * kPT + r) * b + Jt * kPT + c4);
      vb[s][u] = ldcg4(x + (int64_t)(Jt * kPT + r) * b + I * kPT + c4);
    }
  }
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    if (s >= nin) break;
#pragma unroll
    for (int u = 0; u < kQuadSweeps; ++u) {
      const int r = r0 + u * kQuadRows;
      ta[s][r][c4] = va[s][u].x; ta[s][r][c4 + 1] = va[s][u].y;
      ta[s][r][c4 + 2] = va[s][u].z; ta[s][r][c4 + 3] = va[s][u].w;
      tb[s][r][c4] = vb[s][u].x; tb[s][r][c4 + 1] = vb[s][u].y;
      tb[s][r][c4 + 2] = vb[s][u].z; tb[s][r][c4 + 3] = vb[s][u].w;
    }
  }
  __syncthreads();
  const bool two = (I != Jt);
#pragma unroll
  for (int u = 0; u < kQuadSweeps; ++u) {
    const int r = r0 + u * kQuadRows;
    // (X + X^T) at (I*64 + r, J*64 + c) and, for the mirrored tile, (J*64 + r, I*64 + c)
    float v1[2][4], v2[2][4];
#pragma unroll
    for (int s = 0; s < 2; ++s)
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        v1[s][w] = (s < nin) ? ta[s][r][c4 + w] + tb[s][c4 + w][r] : 0.f;
        v2[s][w] = (s < nin) ? tb[s][r][c4 + w] + ta[s][c4 + w][r] : 0.f;
      }
#pragma unroll
    for (int o = 0; o < 4; ++o) {
      if (o >= nout) break;
      float a1[4] = {0.f, 0.f, 0.f, 0.f}, a2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        if (s >= nin) break;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          a1[w] += J.coef[o][s] * v1[s][w];
          a2[w] += J.coef[o][s] * v2[s][w];
        }
      }
      float* y = (o == 0 ? J.C : o == 1 ? J.C2 : J.add_out[o - 2]) + base;
      st4(y + (int64_t)(I * kPT + r) * b + Jt * kPT + c4, a1[0], a1[1], a1[2], a1[3]);
      if (two) st4(y + (int64_t)(Jt * kPT + r) * b + I * kPT + c4, a2[0], a2[1], a2[2], a2[3]);
    }
    if (J.Cb_f) {  // transposed copy: (I,J) <- X_0(J,I)^T, (J,I) <- X_0(I,J)^T
      float* y = J.Cb_f + base;
      st4(y + (int64_t)(I * kPT + r) * b + Jt * kPT + c4, tb[0][c4][r], tb[0][c4 + 1][r],
          tb[0][c4 + 2][r], tb[0][c4 + 3][r]);
      if (two)
        st4(y + (int64_t)(Jt * kPT + r) * b + I * kPT + c4, ta[0][c4][r], ta[0][c4 + 1][r],
            ta[0][c4 + 2][r], ta[0][c4 + 3][r]);
    }
  }
}

// dtheta_idx(i, j) = A_ij - A_ji
template <int NT>
__device__ void pack_tile(const CnpJob& J, int z, int t, int b, float* smem) {
  constexpr int kQuadRows = NT / 16, kQuadSweeps = kPT / kQuadRows;
  static_assert(kQuadRows * kQuadSweeps == kPT, "tile sweep");
  float (*ta)[kPLD] = reinterpret_cast<float (*)[kPLD]>(smem);
  float (*tb)[kPLD] = reinterpret_cast<float (*)[kPLD]>(smem + kPT * kPLD);
  int I, Jt;
  tile_pair(b / kPT, t, I, Jt);
  const float* a = J.A + (int64_t)z * b * b;
  float* th = J.C + z * ((int64_t)b * (b - 1) / 2);
  const int c4 = (threadIdx.x & 15) * 4, r0 = threadIdx.x >> 4;
  float4 va[kQuadSweeps], vb[kQuadSweeps];
#pragma unroll
  for (int u = 0; u < kQuadSweeps; ++u) {
    const int r = r0 + u * kQuadRows;
    va[u] = ldcg4(a + (int64_t)(I * kPT + r) * b + Jt * kPT + c4);
    vb[u] = ldcg4(a + (int64_t)(Jt * kPT + r) * b + I * kPT + c4);
  }
#pragma unroll
  for (int u = 0; u < kQuadSweeps; ++u) {
    const int r = r0 + u * kQuadRows;
    ta[r][c4] = va[u].x; ta[r][c4 + 1] = va[u].y; ta[r][c4 + 2] = va[u].z; ta[r][c4 + 3] = va[u].w;
    tb[r][c4] = vb[u].x; tb[r][c4 + 1] = vb[u].y; tb[r][c4 + 2] = vb[u].z; tb[r][c4 + 3] = vb[u].w;
  }
  __syncthreads();
  // packed rows are contiguous in j but not 16-byte aligned: scalar stores, tx-major
  constexpr int kPRows = NT / kPT;
  const int tx = threadIdx.x & (kPT - 1), ty = threadIdx.x / kPT;
#pragma unroll
  for (int u = 0; u < kPT / kPRows; ++u) {
    const int r = ty + u * kPRows;
    const int i = I * kPT + r, j = Jt * kPT + tx;
    if (i < j) __stcg(th + tri_idx(i, j, b), ta[r][tx] - tb[tx][r]);
  }
}

// ------------------------------------------------------------------ the graph kernel
__device__ __forceinline__ void red_release_add(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

template <int TILE>
__global__ void __launch_bounds__(GraphCfg<TILE>::threads, GraphCfg<TILE>::ctas_per_sm)
    k_cnp_graph(const __grid_constant__ CnpGraph g) {
  constexpr int NT = GraphCfg<TILE>::threads;
  extern __shared__ __align__(16) float smem[];
  __shared__ int s_item, s_next;
  __shared__ int s_ok;
  // the current item's job descriptor, copied from the parameter space once per item so
  // that the tile code reads its fields as shared-memory broadcasts
  __shared__ __align__(16) int s_job[(sizeof(CnpJob) + 3) / 4];
  int* ticket = g.counters + g.njobs * g.nblk;
  const int total = g.item_start[g.njobs];
  pdl_trigger();
  pdl_wait();
  // three single-thread roles per item, in different warps so that none waits on another:
  // thread 0 checks the item's dependencies, thread 32 takes the next ticket, thread 64
  // publishes the previous item's completion
  constexpr int kTicketThread = 32, kReleaseThread = 64;
  int done_job = -1, done_z = 0;  // the previous item, published at the next item's start
  if (threadIdx.x == kTicketThread) s_next = atomicAdd(ticket, 1);
  for (;;) {
    __syncthreads();  // smem of the previous item is free; s_next is visible
    if (threadIdx.x == 0) {
      s_item = s_next;
      s_ok = 1;
    }
    __syncthreads();
    // publish the previous item: the two barriers order every thread's stores of it before
    // this release, which waits on nothing, so a published item is never held up by the
    // next item's dependencies
    if (threadIdx.x == kReleaseThread && done_job >= 0)
      red_release_add(g.counters + done_job * g.nblk + done_z, 1);
    const int item = s_item;
    if (item >= total) break;
    int j = 0;
    while (item >= g.item_start[j + 1]) ++j;
    {
      const int* src = reinterpret_cast<const int*>(&g.job[j]);
      for (int w = threadIdx.x; w < (int)(sizeof(CnpJob) / 4); w += blockDim.x) s_job[w] = src[w];
    }
    const int tiles = g.job[j].tiles;
    const int local = item - g.item_start[j];
    const int z = local / tiles;
    const int t = local - z * tiles;
    const unsigned deps = g.job[j].deps;
    // next ticket in flight while this item runs
    if (threadIdx.x == kTicketThread) s_next = atomicAdd(ticket, 1);
    if (threadIdx.x == 0) {
      // wait until every job this one reads has finished for block z
      const unsigned long long t0 = gtimer();
      for (int d = 0; d < j && s_ok; ++d) {
        if (!((deps >> d) & 1u)) continue;
        const int* cnt = g.counters + d * g.nblk + z;
        const int need = g.job[d].tiles;
        unsigned spins = 0;
        while (ld_acquire(cnt) < need) {
          if ((++spins & 31u) == 0) {
            if (*reinterpret_cast<volatile int*>(g.err) != 0 ||
                gtimer() - t0 > g.wait_ns) {
              atomicCAS(g.err, 0, (int)POETX_ERR_TIMEOUT);
              s_ok = 0;
              break;
            }
            __nanosleep(64);
          }
        }
      }
    }
    __syncthreads();  // also publishes s_job
    if (!s_ok) break;
    const CnpJob& J = *reinterpret_cast<const CnpJob*>(s_job);
    switch (J.type) {
      case JOB_EXPAND: expand_tile<NT>(J, z, t, g.b, smem); break;
      case JOB_PRODUCT:
        if (TILE == 64)
          product_tile64(J, z, t, g.b, smem);
        else
          product_tile128(J, z, t, g.b, smem);
        break;
      case JOB_SYMCOMB: symcomb_tile<NT>(J, z, t, g.b, smem); break;
      default: pack_tile<NT>(J, z, t, g.b, smem); break;
    }
    done_job = j;
    done_z = z;
  }
}

// p[0] = first, p[1..n) = 0
__global__ void k_zero_ints(int* p, int n, int first) {
  pdl_trigger();
  pdl_wait();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
    p[i] = i == 0 ? first : 0;
}

// items per block of a job: output tiles of a product (tile x tile; upper tiles only for
// symmetric results), 64 x 64 tile pairs of an elementwise job
int cnp_graph_tiles(int type, int mode, int b, int tile) {
  if (type == JOB_PRODUCT) {
    const int nt = b / tile;
    return mode == SG_FULL ? nt * nt : nt * (nt + 1) / 2;
  }
  const int nt = b / 64;
  return nt * (nt + 1) / 2;
}

template <int TILE>
cudaError_t launch_graph_t(const CnpGraph& g, cudaStream_t s) {
  using Cfg = GraphCfg<TILE>;
  // persistent grid: never more CTAs than can be resident at once
  static int per_sm_dev[64] = {0};  // once per device, outside any stream capture
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  int& per_sm = per_sm_dev[dev];
  cudaError_t e;
  if (per_sm == 0) {
    int v = 0;
    e = cudaFuncSetAttribute(k_cnp_graph<TILE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg::smem);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, k_cnp_graph<TILE>, Cfg::threads,
                                                      Cfg::smem);
    if (e != cudaSuccess) return e;
    per_sm = v > 0 ? v : 1;
  }
  int grid = num_sms() * per_sm;
  const int total = g.item_start[g.njobs];
  if (grid > total) grid = total;
  begin_launch("cnp_sgemm", s);
  e = launch_pdl(k_cnp_graph<TILE>, dim3(grid), dim3(Cfg::threads), Cfg::smem, s, g);
  end_launch("cnp_sgemm", s);
  return e;
}

}  // namespace

cudaError_t launch_cnp_graph(CnpGraph g, cudaStream_t s) {
  if (g.njobs <= 0 || g.nblk <= 0) return cudaSuccess;
  for (int j = 0; j < g.njobs; ++j) {  // shapes the tile code relies on
    const CnpJob& J = g.job[j];
    if (J.type == JOB_PRODUCT && J.nadd + (J.skew_add ? 1 : 0) > kEpiTiles)
      return cudaErrorInvalidValue;
    if (J.type == JOB_PRODUCT && J.A2 && J.alpha2 != 1.f && J.alpha2 != -1.f)
      return cudaErrorInvalidValue;
    if (J.type == JOB_SYMCOMB && (J.nin < 1 || J.nin > 2 || J.nout < 1 || J.nout > 4))
      return cudaErrorInvalidValue;
  }
  // 128 x 128 product items when every level of the chain has at least two waves of them
  // (two CTAs per SM); otherwise 64 x 64 items, which split a block four times finer
  const int nt128 = g.b % 128 == 0 ? g.b / 128 : 0;
  const int sym_items = g.nblk * nt128 * (nt128 + 1) / 2;
  const int tile = (nt128 > 0 && sym_items >= 4 * num_sms()) ? 128 : 64;
  g.item_start[0] = 0;
  for (int j = 0; j < g.njobs; ++j) {
    g.job[j].tiles = cnp_graph_tiles(g.job[j].type, g.job[j].mode, g.b, tile);
    g.item_start[j + 1] = g.item_start[j] + g.job[j].tiles * g.nblk;
  }
  g.err = device_error_flag();
  if (!g.err) return cudaErrorInvalidDevice;  // the bounded waits need the flag
  g.wait_ns = wait_limit_ns();
  const int ncount = g.njobs * g.nblk + 1;
  begin_launch("cnp_elementwise", s);
  cudaError_t e = launch_pdl(k_zero_ints, dim3((ncount + 255) / 256), dim3(256), 0, s,
                             g.counters, ncount, g.first_counter);
  end_launch("cnp_elementwise", s);
  if (e != cudaSuccess) return e;
  return tile == 128 ? launch_graph_t<128>(g, s) : launch_graph_t<64>(g, s);
}

}  // namespace poetx
