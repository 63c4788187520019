// fp32 SIMT kernels: a batched FFMA GEMM with structured (symmetric / symmetric+skew)
// outputs, and the small elementwise kernels of the Cayley-Neumann parameterisation
// (POET-X technical summary, section 2.4).  They run the fp32 layer and the CNP shapes
// outside the one-launch task graph (b % 64 != 0 or more than three powers of S), plus
// the fixed-order reduction of split token sums.
//
// The CNP works on b x b blocks in fp32.  Its products are between polynomials in the
// skew-symmetric Q, so most outputs are symmetric (even powers of Q) or skew (odd
// powers): for those only the tiles on and above the diagonal are computed and the
// mirror half is written from the same registers, halving the FFMA work.
#include <cuda_bf16.h>

#include "poetx_internal.h"

namespace poetx {
namespace {

constexpr int kThreads = 256;  // 16 x 16 thread grid

struct SgemmDev {
  const float* A;
  int64_t lda, sA;
  const float* B;
  int64_t ldb, sB;
  int transA, transB;
  const float* A2;
  int64_t lda2, sA2;
  const float* B2;
  int64_t ldb2, sB2;
  int transA2, transB2;
  int K2;
  float alpha2;
  float* C;
  int64_t ldc, sC;
  __nv_bfloat16* Cb;
  float* C2;
  float alpha_c2, diag2;
  float addc2[8];
  int M, N, K, batch;
  float alpha;
  int nadd;
  const float* add[8];
  float addc[8];
  const float* skew_add;
  float skew_c;
  float diag;
  int mode;
  int tiles_per_batch;
  int tiles_n;  // FULL mode
  int nt;       // structured modes: tiles per side
};

// Thread (tx, ty) owns rows g*(16*VEC) + ty*VEC + v and the same pattern of columns.
template <int TM, int BK>
struct Tile {
  static constexpr int VEC = TM < 4 ? TM : 4;
  static constexpr int NG = TM / VEC;
  static constexpr int BM = 16 * TM;
  static constexpr int LOADS = BM * BK / kThreads;  // elements per thread per operand tile
  // the mirror half of SYM / SYMSKEW tiles is staged in smem when it fits the A buffers
  static constexpr bool STAGE = (BM * (BM + 1)) <= 2 * BK * (BM + 4);
};

template <int TM, int BK>
__device__ __forceinline__ void load_tile_regs(float (&r)[Tile<TM, BK>::LOADS], const float* X,
                                               int64_t ldx, int trans, int row0, int k0,
                                               int rows, int kdim, float scale, bool is_b) {
  // Loads the (BM x BK) tile of op(X) (for A) or the (BK x BN) tile of op(B), as
  // element (row, k) with row in [row0, row0+BM), k in [k0, k0+BK).
  // A: op(A)[i][k] = trans ? X[k*ld + i] : X[i*ld + k]
  // B: op(B)[k][j] = trans ? X[j*ld + k] : X[k*ld + j]   (j plays the role of row)
  constexpr int BM = Tile<TM, BK>::BM;
  const int tid = threadIdx.x;
  const bool k_contig = is_b ? (trans != 0) : (trans == 0);
#pragma unroll
  for (int l = 0; l < Tile<TM, BK>::LOADS; ++l) {
    int idx = tid + l * kThreads;
    int i, k;
    if (k_contig) {
      i = idx / BK;
      k = idx % BK;
    } else {
      k = idx / BM;
      i = idx % BM;
    }
    int gi = row0 + i, gk = k0 + k;
    float v = 0.f;
    if (gi < rows && gk < kdim) {
      int64_t off = k_contig ? ((int64_t)gi * ldx + gk) : ((int64_t)gk * ldx + gi);
      v = __ldg(X + off) * scale;
    }
    r[l] = v;
  }
}

template <int TM, int BK>
__device__ __forceinline__ void store_tile_smem(const float (&r)[Tile<TM, BK>::LOADS],
                                                float (*S)[Tile<TM, BK>::BM + 4], int trans,
                                                bool is_b) {
  constexpr int BM = Tile<TM, BK>::BM;
  const int tid = threadIdx.x;
  const bool k_contig = is_b ? (trans != 0) : (trans == 0);
#pragma unroll
  for (int l = 0; l < Tile<TM, BK>::LOADS; ++l) {
    int idx = tid + l * kThreads;
    int i, k;
    if (k_contig) {
      i = idx / BK;
      k = idx % BK;
    } else {
      k = idx / BM;
      i = idx % BM;
    }
    S[k][i] = r[l];
  }
}

template <int TM, int BK>
__global__ void __launch_bounds__(kThreads, TM <= 4 ? 2 : 1) k_sgemm(SgemmDev p) {
  using TL = Tile<TM, BK>;
  constexpr int BM = TL::BM, VEC = TL::VEC, NG = TL::NG;
  __shared__ __align__(16) float As[2][BK][BM + 4];
  __shared__ __align__(16) float Bs[2][BK][BM + 4];

  const int tile_lin = blockIdx.x;
  const int bz = tile_lin / p.tiles_per_batch;
  int t = tile_lin - bz * p.tiles_per_batch;
  int I, J;
  if (p.mode == SG_FULL) {
    I = t / p.tiles_n;
    J = t - I * p.tiles_n;
  } else {
    I = 0;
    while (t >= p.nt - I) {
      t -= p.nt - I;
      ++I;
    }
    J = I + t;
  }
  const int m0 = I * BM, n0 = J * BM;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;

  float acc[TM][TM];
#pragma unroll
  for (int a = 0; a < TM; ++a)
#pragma unroll
    for (int c = 0; c < TM; ++c) acc[a][c] = 0.f;

  float ra[TL::LOADS], rb[TL::LOADS];
  const int nk1 = (p.K + BK - 1) / BK;
  const int nk2 = p.A2 ? (p.K2 + BK - 1) / BK : 0;
  const int nkt = nk1 + nk2;

  auto load = [&](int kt) {
    if (kt < nk1) {
      load_tile_regs<TM, BK>(ra, p.A + bz * p.sA, p.lda, p.transA, m0, kt * BK, p.M, p.K, 1.f,
                             false);
      load_tile_regs<TM, BK>(rb, p.B + bz * p.sB, p.ldb, p.transB, n0, kt * BK, p.N, p.K, 1.f,
                             true);
    } else {
      int k2 = (kt - nk1) * BK;
      load_tile_regs<TM, BK>(ra, p.A2 + bz * p.sA2, p.lda2, p.transA2, m0, k2, p.M, p.K2,
                             p.alpha2, false);
      load_tile_regs<TM, BK>(rb, p.B2 + bz * p.sB2, p.ldb2, p.transB2, n0, k2, p.N, p.K2, 1.f,
                             true);
    }
  };
  auto store = [&](int kt, int buf) {
    int ta = kt < nk1 ? p.transA : p.transA2;
    int tb = kt < nk1 ? p.transB : p.transB2;
    store_tile_smem<TM, BK>(ra, As[buf], ta, false);
    store_tile_smem<TM, BK>(rb, Bs[buf], tb, true);
  };

  if (nkt > 0) {
    load(0);
    store(0, 0);
  }
  __syncthreads();
  for (int kt = 0; kt < nkt; ++kt) {
    const int buf = kt & 1;
    if (kt + 1 < nkt) load(kt + 1);
#pragma unroll
    for (int k = 0; k < BK; ++k) {
      float a[TM], b[TM];
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        if constexpr (VEC == 4) {
          float4 va = *reinterpret_cast<const float4*>(&As[buf][k][g * 16 * VEC + ty * VEC]);
          float4 vb = *reinterpret_cast<const float4*>(&Bs[buf][k][g * 16 * VEC + tx * VEC]);
          a[g * 4 + 0] = va.x; a[g * 4 + 1] = va.y; a[g * 4 + 2] = va.z; a[g * 4 + 3] = va.w;
          b[g * 4 + 0] = vb.x; b[g * 4 + 1] = vb.y; b[g * 4 + 2] = vb.z; b[g * 4 + 3] = vb.w;
        } else {
#pragma unroll
          for (int v = 0; v < VEC; ++v) {
            a[g * VEC + v] = As[buf][k][g * 16 * VEC + ty * VEC + v];
            b[g * VEC + v] = Bs[buf][k][g * 16 * VEC + tx * VEC + v];
          }
        }
      }
#pragma unroll
      for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TM; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    if (kt + 1 < nkt) store(kt + 1, buf ^ 1);
    __syncthreads();
  }

  // ---- epilogue
  const int64_t boff = (int64_t)bz * p.sC;
  float* C = p.C + boff;
  __nv_bfloat16* Cb = p.Cb ? p.Cb + boff : nullptr;
  float* C2 = p.C2 ? p.C2 + boff : nullptr;
  const bool structured = p.mode != SG_FULL;
  // mirror half staged in smem (coalesced transposed store), when the tile fits
  constexpr bool STAGE = TL::STAGE;
  float (*Ms)[BM + 1] = reinterpret_cast<float (*)[BM + 1]>(&As[0][0][0]);
  float (*Ms2)[BM + 1] = reinterpret_cast<float (*)[BM + 1]>(&Bs[0][0][0]);
#pragma unroll
  for (int gi = 0; gi < NG; ++gi)
#pragma unroll
    for (int vi = 0; vi < VEC; ++vi) {
      const int il = gi * 16 * VEC + ty * VEC + vi;
      const int i = m0 + il;
#pragma unroll
      for (int gj = 0; gj < NG; ++gj)
#pragma unroll
        for (int vj = 0; vj < VEC; ++vj) {
          const int jl = gj * 16 * VEC + tx * VEC + vj;
          const int j = n0 + jl;
          if (i >= p.M || j >= p.N) continue;
          if (structured && I == J && i > j) continue;  // mirror of (j, i)
          const int64_t ij = (int64_t)i * p.ldc + j;
          const float a = acc[gi * VEC + vi][gj * VEC + vj];
          float sym = (i == j) ? p.diag : 0.f;
          float sym2 = (i == j) ? p.diag2 : 0.f;
          for (int q = 0; q < p.nadd; ++q) {
            const float x = p.add[q][boff + ij];
            sym += p.addc[q] * x;
            sym2 += p.addc2[q] * x;
          }
          float skew = p.alpha * a;
          if (p.skew_add) skew += p.skew_c * p.skew_add[boff + ij];
          float v, vm, v2 = 0.f;
          if (p.mode == SG_SYMSKEW) {
            v = (i == j) ? sym : sym + skew;   // G_ij = E_ij + O_ij (O_ii = 0)
            vm = sym - skew;                   // G_ji = E_ij - O_ij
          } else {
            v = skew + sym;
            vm = v;
            v2 = p.alpha_c2 * a + sym2;
          }
          C[ij] = v;
          if (Cb) Cb[ij] = __float2bfloat16_rn(v);
          if (C2 && !(p.mode == SG_SYMSKEW)) C2[ij] = v2;
          if (structured && i != j) {
            if constexpr (STAGE) {
              Ms[il][jl] = vm;
              if (C2) Ms2[il][jl] = v2;
            } else {
              const int64_t ji = (int64_t)j * p.ldc + i;
              C[ji] = vm;
              if (Cb) Cb[ji] = __float2bfloat16_rn(vm);
              if (C2) C2[ji] = v2;
            }
          }
        }
    }
  if constexpr (STAGE) {
    if (structured) {
      __syncthreads();
      // C[n0 + jl][m0 + il] = Ms[il][jl] for the strictly-upper part of the tile
      for (int e = threadIdx.x; e < BM * BM; e += kThreads) {
        const int jl = e / BM, il = e - jl * BM;
        const int i = m0 + il, j = n0 + jl;
        if (i >= p.M || j >= p.N) continue;
        if (I == J && il >= jl) continue;
        const int64_t ji = (int64_t)j * p.ldc + i;
        const float vm = Ms[il][jl];
        C[ji] = vm;
        if (Cb) Cb[ji] = __float2bfloat16_rn(vm);
        if (C2) C2[ji] = Ms2[il][jl];
      }
    }
  }
}

// ---- square-block products (b % 64 == 0, no transposes): the CNP's workhorse ---------
// 64 x 64 output tile per CTA, 128 threads, thread (tx = tid & 15, ty = tid >> 4) owns rows
// ty*8 .. ty*8+7 and columns tx*4 .. tx*4+3.  K tiles of 16, register-prefetched.  No
// bounds checks: every tile is full.  A symmetric or skew A (a_sym = +-1) is read by rows
// as its own transpose, so both operands go to shared memory with 16-byte stores.
constexpr int kMMThreads = 128;
constexpr int kMMBK = 16;
constexpr int kMMLD = 64 + 4;

struct MMSmem {
  float As[2][kMMBK][kMMLD];
  float Bs[2][kMMBK][kMMLD];
};
constexpr int kMMStage = 2 * 64 * 65;  // two 64 x 65 staging tiles for the mirror half
constexpr int kMMStages = 4;            // cp.async ring depth of the row-operand path
constexpr int kMMStageFloats = 2 * kMMBK * kMMLD;
constexpr int kMMSmemFloats = kMMStages * kMMStageFloats > kMMStage
                                  ? kMMStages * kMMStageFloats : kMMStage;

__device__ __forceinline__ void mm_cp_async16(float* smem_dst, const float* gsrc) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void mm_cp_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void mm_cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ float4 ldg4(const float* p) {
  return __ldg(reinterpret_cast<const float4*>(p));
}

// ROWS: every A operand of the launch is readable by rows (symmetric, skew, or given as
// its transpose), so A and B tiles stream through a 4-deep cp.async ring; the sign of a
// skew operand and alpha2 = -1 are applied to the accumulators (acc_scale below).
// !ROWS: register-staged loads with a transposing store for a general A.
template <bool ROWS>
__global__ void __launch_bounds__(kMMThreads, 4) k_cnp_mm(SgemmDev p, int a_sym, int a2_sym) {
  __shared__ __align__(16) float smem[kMMSmemFloats];
  MMSmem& S = *reinterpret_cast<MMSmem*>(smem);
  (void)S;
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;

  const int bz = blockIdx.x / p.tiles_per_batch;
  int t = blockIdx.x - bz * p.tiles_per_batch;
  int I, J;
  if (p.mode == SG_FULL) {
    I = t / p.tiles_n;
    J = t - I * p.tiles_n;
  } else {
    I = 0;
    while (t >= p.nt - I) {
      t -= p.nt - I;
      ++I;
    }
    J = I + t;
  }
  const int m0 = I * 64, n0 = J * 64;
  const int b = p.ldc;  // square blocks: ld = b for every operand

  float acc[8][4];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;

  const int nk1 = p.K / kMMBK;
  const int nk2 = p.A2 ? p.K2 / kMMBK : 0;
  const int nkt = nk1 + nk2;

  // multiplier that turns the accumulators into op(A) op(B) + alpha2 op(A2) op(B2)
  float acc_scale = 1.f;
  if constexpr (ROWS) {
    const float s1 = a_sym < 0 ? -1.f : 1.f;
    const float s2 = a2_sym < 0 ? -1.f : 1.f;
    const float boundary = s1 * s2 * p.alpha2;  // applied before the second product
    acc_scale = nk2 > 0 ? s2 * p.alpha2 : s1;
    auto As_ = [&](int st) {
      return reinterpret_cast<float (*)[kMMLD]>(smem + st * kMMStageFloats);
    };
    auto Bs_ = [&](int st) {
      return reinterpret_cast<float (*)[kMMLD]>(smem + st * kMMStageFloats + kMMBK * kMMLD);
    };
    auto issue = [&](int kt) {
      if (kt < nkt) {
        const bool first = kt < nk1;
        const float* A = first ? p.A + bz * p.sA : p.A2 + bz * p.sA2;
        const float* B = first ? p.B + bz * p.sB : p.B2 + bz * p.sB2;
        const int k0 = (first ? kt : kt - nk1) * kMMBK;
        const int st = kt % kMMStages;
        float (*As)[kMMLD] = As_(st);
        float (*Bs)[kMMLD] = Bs_(st);
#pragma unroll
        for (int l = 0; l < 2; ++l) {
          const int f = tid + l * kMMThreads;
          const int r = f >> 4, c4 = (f & 15) * 4;
          mm_cp_async16(&As[r][c4], A + (int64_t)(k0 + r) * b + m0 + c4);
          mm_cp_async16(&Bs[r][c4], B + (int64_t)(k0 + r) * b + n0 + c4);
        }
      }
      mm_cp_commit();
    };
#pragma unroll
    for (int st = 0; st < kMMStages - 1; ++st) issue(st);
    for (int kt = 0; kt < nkt; ++kt) {
      mm_cp_wait<kMMStages - 2>();
      __syncthreads();
      issue(kt + kMMStages - 1);
      if (nk2 > 0 && kt == nk1) {
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[r][c] *= boundary;
      }
      const int st = kt % kMMStages;
      float (*As)[kMMLD] = As_(st);
      float (*Bs)[kMMLD] = Bs_(st);
#pragma unroll
      for (int k = 0; k < kMMBK; ++k) {
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
    }
    mm_cp_wait<0>();
    __syncthreads();
  } else {
  float4 ra[2], rb[2];
  // global -> registers for k tile kt
  auto load = [&](int kt) {
    const bool first = kt < nk1;
    const float* A = first ? p.A + bz * p.sA : p.A2 + bz * p.sA2;
    const float* B = first ? p.B + bz * p.sB : p.B2 + bz * p.sB2;
    const int k0 = (first ? kt : kt - nk1) * kMMBK;
    const int sym = (first ? a_sym : a2_sym) == 2 ? 1 : (first ? a_sym : a2_sym);
    const float sc = first ? 1.f : p.alpha2;
#pragma unroll
    for (int l = 0; l < 2; ++l) {
      const int f = tid + l * kMMThreads;  // 0..255
      // B tile: 16 rows (k) x 64 cols, 16 float4 per row
      const int br = f >> 4, bc = (f & 15) * 4;
      rb[l] = ldg4(B + (int64_t)(k0 + br) * b + n0 + bc);
      float4 a;
      if (sym != 0) {  // As[k][i] = sym * A[k][i]: rows of A are its transpose's columns
        a = ldg4(A + (int64_t)(k0 + br) * b + m0 + bc);
        const float s2 = sc * (float)sym;
        a.x *= s2; a.y *= s2; a.z *= s2; a.w *= s2;
      } else {         // As[k][i] = A[i][k]: 64 rows x 4 float4 of k
        const int ar = f >> 2, ac = (f & 3) * 4;
        a = ldg4(A + (int64_t)(m0 + ar) * b + k0 + ac);
        a.x *= sc; a.y *= sc; a.z *= sc; a.w *= sc;
      }
      ra[l] = a;
    }
  };
  auto store = [&](int kt, int buf) {
    const int sym = kt < nk1 ? a_sym : a2_sym;
#pragma unroll
    for (int l = 0; l < 2; ++l) {
      const int f = tid + l * kMMThreads;
      const int br = f >> 4, bc = (f & 15) * 4;
      *reinterpret_cast<float4*>(&S.Bs[buf][br][bc]) = rb[l];
      if (sym != 0) {
        *reinterpret_cast<float4*>(&S.As[buf][br][bc]) = ra[l];
      } else {
        const int ar = f >> 2, ac = (f & 3) * 4;
        S.As[buf][ac + 0][ar] = ra[l].x;
        S.As[buf][ac + 1][ar] = ra[l].y;
        S.As[buf][ac + 2][ar] = ra[l].z;
        S.As[buf][ac + 3][ar] = ra[l].w;
      }
    }
  };

  if (nkt > 0) {
    load(0);
    store(0, 0);
  }
  __syncthreads();
  for (int kt = 0; kt < nkt; ++kt) {
    const int buf = kt & 1;
    if (kt + 1 < nkt) load(kt + 1);
#pragma unroll
    for (int k = 0; k < kMMBK; ++k) {
      const float4 a0 = *reinterpret_cast<const float4*>(&S.As[buf][k][ty * 8]);
      const float4 a1 = *reinterpret_cast<const float4*>(&S.As[buf][k][ty * 8 + 4]);
      const float4 bv = *reinterpret_cast<const float4*>(&S.Bs[buf][k][tx * 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bb[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(a[r], bb[c], acc[r][c]);
    }
    if (kt + 1 < nkt) store(kt + 1, buf ^ 1);
    __syncthreads();
  }
  }  // !ROWS

  // ---- epilogue (same semantics as k_sgemm)
  const int64_t boff = (int64_t)bz * p.sC;
  float* C = p.C + boff;
  __nv_bfloat16* Cb = p.Cb ? p.Cb + boff : nullptr;
  float* C2 = p.C2 ? p.C2 + boff : nullptr;
  const bool structured = p.mode != SG_FULL;
  float (*Ms)[65] = reinterpret_cast<float (*)[65]>(smem);
  float (*Ms2)[65] = reinterpret_cast<float (*)[65]>(smem + 64 * 65);
  const int jl0 = tx * 4;
  const int j0 = n0 + jl0;
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int il = ty * 8 + r;
    const int i = m0 + il;
    const int64_t row = (int64_t)i * b;
    float sym[4] = {0.f, 0.f, 0.f, 0.f}, sym2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < 4; ++c)
      if (i == j0 + c) {
        sym[c] = p.diag;
        sym2[c] = p.diag2;
      }
    for (int q = 0; q < p.nadd; ++q) {
      const float4 x = ldg4(p.add[q] + boff + row + j0);
      const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        sym[c] += p.addc[q] * xs[c];
        sym2[c] += p.addc2[q] * xs[c];
      }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[r][c] *= acc_scale;
    float skew[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) skew[c] = p.alpha * acc[r][c];
    if (p.skew_add) {
      const float4 x = ldg4(p.skew_add + boff + row + j0);
      skew[0] += p.skew_c * x.x; skew[1] += p.skew_c * x.y;
      skew[2] += p.skew_c * x.z; skew[3] += p.skew_c * x.w;
    }
    float v[4], vm[4], v2[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = j0 + c;
      if (p.mode == SG_SYMSKEW) {
        v[c] = (i == j) ? sym[c] : sym[c] + skew[c];
        vm[c] = sym[c] - skew[c];
      } else {
        v[c] = skew[c] + sym[c];
        vm[c] = v[c];
      }
      v2[c] = p.alpha_c2 * acc[r][c] + sym2[c];
    }
    // in diagonal tiles of structured outputs only the upper triangle is written here
    if (structured && I == J) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int j = j0 + c;
        if (i <= j) {
          C[row + j] = v[c];
          if (Cb) Cb[row + j] = __float2bfloat16_rn(v[c]);
          if (C2) C2[row + j] = v2[c];
        }
      }
    } else {
      *reinterpret_cast<float4*>(C + row + j0) = make_float4(v[0], v[1], v[2], v[3]);
      if (Cb) {
        __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]);
        __nv_bfloat162 h1 = __floats2bfloat162_rn(v[2], v[3]);
        uint2 o;
        o.x = *reinterpret_cast<uint32_t*>(&h0);
        o.y = *reinterpret_cast<uint32_t*>(&h1);
        *reinterpret_cast<uint2*>(Cb + row + j0) = o;
      }
      if (C2) *reinterpret_cast<float4*>(C2 + row + j0) = make_float4(v2[0], v2[1], v2[2], v2[3]);
    }
    if (structured) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        Ms[il][jl0 + c] = vm[c];
        if (C2) Ms2[il][jl0 + c] = v2[c];
      }
    }
  }
  if (structured) {
    // the main loop ended with a barrier, so the staging tiles may overwrite As/Bs; one
    // more barrier makes every thread's staged values visible
    __syncthreads();
    for (int e = tid; e < 64 * 64; e += kMMThreads) {
      const int jl = e >> 6, il = e & 63;
      if (I == J && il >= jl) continue;
      const int64_t ji = (int64_t)(n0 + jl) * b + m0 + il;
      const float vmv = Ms[il][jl];
      C[ji] = vmv;
      if (Cb) Cb[ji] = __float2bfloat16_rn(vmv);
      if (C2) C2[ji] = Ms2[il][jl];
    }
  }
}

// ---- tile-pair elementwise kernels (32 x 32 tiles, I <= J) --------------------------

__device__ __forceinline__ void tile_pair(int nt, int t, int& I, int& J) {
  I = 0;
  while (t >= nt - I) {
    t -= nt - I;
    ++I;
  }
  J = I + t;
}

__device__ __forceinline__ int64_t tri_idx(int i, int j, int b) {
  // strict upper triangle, row-major: idx(i,j) = i*b - i*(i+1)/2 + (j-i-1), i < j
  return (int64_t)i * b - (int64_t)i * (i + 1) / 2 + (j - i - 1);
}

__global__ void __launch_bounds__(256) k_theta_to_Q(const float* __restrict__ theta,
                                                    float* __restrict__ Q, int b, int nt,
                                                    int pairs) {
  __shared__ float t[32][33];
  const int blk = blockIdx.x / pairs;
  int I, J;
  tile_pair(nt, blockIdx.x - blk * pairs, I, J);
  const int64_t ntri = (int64_t)b * (b - 1) / 2;
  const float* th = theta + blk * ntri;
  float* q = Q + (int64_t)blk * b * b;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int r = ty; r < 32; r += 8) {
    int i = I * 32 + r, j = J * 32 + tx;
    t[r][tx] = (i < b && j < b && i < j) ? th[tri_idx(i, j, b)] : 0.f;
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    int i = I * 32 + r, j = J * 32 + tx;
    if (i < b && j < b) q[(int64_t)i * b + j] = (I == J && r > tx) ? -t[tx][r] : t[r][tx];
  }
  if (I != J) {
    for (int r = ty; r < 32; r += 8) {
      int i = J * 32 + r, j = I * 32 + tx;
      if (i < b && j < b) q[(int64_t)i * b + j] = -t[tx][r];
    }
  }
}

struct SymcombDev {
  const float* X[4];
  float* out[4];
  float coef[4][4];
  int nin, nout;
  float* tout;  // optional: tout = X[0]^T
};

__global__ void __launch_bounds__(256) k_symcomb(SymcombDev p, int b, int nt, int pairs) {
  __shared__ float ta[32][33], tb[32][33];
  __shared__ float acc[4][32][33];
  const int blk = blockIdx.x / pairs;
  int I, J;
  tile_pair(nt, blockIdx.x - blk * pairs, I, J);
  const int64_t base = (int64_t)blk * b * b;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int o = 0; o < p.nout; ++o)
    for (int r = ty; r < 32; r += 8) acc[o][r][tx] = 0.f;
  for (int s = 0; s < p.nin; ++s) {
    const float* x = p.X[s] + base;
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {
      int i = I * 32 + r, j = J * 32 + tx;
      ta[r][tx] = (i < b && j < b) ? x[(int64_t)i * b + j] : 0.f;
      int i2 = J * 32 + r, j2 = I * 32 + tx;
      tb[r][tx] = (i2 < b && j2 < b) ? x[(int64_t)i2 * b + j2] : 0.f;
    }
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {
      float v = ta[r][tx] + tb[tx][r];  // (X + X^T)[I*32 + r, J*32 + tx]
      for (int o = 0; o < p.nout; ++o) acc[o][r][tx] += p.coef[o][s] * v;
    }
    if (s == 0 && p.tout) {  // transposed copy: tout(I,J) = X(J,I)^T, tout(J,I) = X(I,J)^T
      float* y = p.tout + base;
      for (int r = ty; r < 32; r += 8) {
        int i = I * 32 + r, j = J * 32 + tx;
        if (i < b && j < b) y[(int64_t)i * b + j] = tb[tx][r];
        int i2 = J * 32 + r, j2 = I * 32 + tx;
        if (I != J && i2 < b && j2 < b) y[(int64_t)i2 * b + j2] = ta[tx][r];
      }
    }
  }
  __syncthreads();
  for (int o = 0; o < p.nout; ++o) {
    float* y = p.out[o] + base;
    for (int r = ty; r < 32; r += 8) {
      int i = I * 32 + r, j = J * 32 + tx;
      if (i < b && j < b && !(I == J && r > tx)) y[(int64_t)i * b + j] = acc[o][r][tx];
      if (I == J && r > tx && i < b && j < b) y[(int64_t)i * b + j] = acc[o][tx][r];
    }
    if (I != J) {
      for (int r = ty; r < 32; r += 8) {
        int i = J * 32 + r, j = I * 32 + tx;
        if (i < b && j < b) y[(int64_t)i * b + j] = acc[o][tx][r];
      }
    }
  }
}

__global__ void __launch_bounds__(256) k_pack_skew(const float* __restrict__ A,
                                                   float* __restrict__ dtheta, int b, int nt,
                                                   int pairs) {
  __shared__ float ta[32][33], tb[32][33];
  const int blk = blockIdx.x / pairs;
  int I, J;
  tile_pair(nt, blockIdx.x - blk * pairs, I, J);
  const float* a = A + (int64_t)blk * b * b;
  float* th = dtheta + (int64_t)blk * ((int64_t)b * (b - 1) / 2);
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int r = ty; r < 32; r += 8) {
    int i = I * 32 + r, j = J * 32 + tx;
    ta[r][tx] = (i < b && j < b) ? a[(int64_t)i * b + j] : 0.f;
    int i2 = J * 32 + r, j2 = I * 32 + tx;
    tb[r][tx] = (i2 < b && j2 < b) ? a[(int64_t)i2 * b + j2] : 0.f;
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    int i = I * 32 + r, j = J * 32 + tx;
    if (i < b && j < b && i < j) th[tri_idx(i, j, b)] = ta[r][tx] - tb[tx][r];
  }
}

__global__ void k_split_reduce(const float* __restrict__ src, int nsplit, int64_t stride,
                               float* __restrict__ dst, int64_t count, int accumulate) {
  pdl_trigger();
  pdl_wait();
  const int64_t n4 = count / 4;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    float4 acc = accumulate ? reinterpret_cast<const float4*>(dst)[i] : make_float4(0, 0, 0, 0);
    // the first kBatch partials are all loaded before any is added (one memory round trip
    // instead of one per partial); the sum keeps the split order, so results are unchanged
    constexpr int kBatch = 16;
    float4 v[kBatch];
#pragma unroll
    for (int s = 0; s < kBatch; ++s)
      if (s < nsplit) v[s] = __ldg(reinterpret_cast<const float4*>(src + s * stride) + i);
#pragma unroll
    for (int s = 0; s < kBatch; ++s) {
      if (s < nsplit) {
        acc.x += v[s].x; acc.y += v[s].y; acc.z += v[s].z; acc.w += v[s].w;
      }
    }
    for (int s = kBatch; s < nsplit; ++s) {
      const float4 u = __ldg(reinterpret_cast<const float4*>(src + s * stride) + i);
      acc.x += u.x; acc.y += u.y; acc.z += u.z; acc.w += u.w;
    }
    reinterpret_cast<float4*>(dst)[i] = acc;
  }
  for (int64_t i = n4 * 4 + blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count;
       i += (int64_t)gridDim.x * blockDim.x) {
    float acc = accumulate ? dst[i] : 0.f;
    for (int s = 0; s < nsplit; ++s) acc += src[s * stride + i];
    dst[i] = acc;
  }
}

__global__ void k_f32_to_bf16(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                              int64_t count) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count;
       i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = __float2bfloat16_rn(src[i]);
}

int ceil_div(int a, int b) { return (a + b - 1) / b; }

SgemmDev make_dev(const SgemmArgs& a) {
  SgemmDev p;
  p.A = a.A; p.lda = a.lda; p.sA = a.sA;
  p.B = a.B; p.ldb = a.ldb; p.sB = a.sB;
  p.transA = a.transA; p.transB = a.transB;
  p.A2 = a.A2; p.lda2 = a.lda2; p.sA2 = a.sA2;
  p.B2 = a.B2; p.ldb2 = a.ldb2; p.sB2 = a.sB2;
  p.transA2 = a.transA2; p.transB2 = a.transB2;
  p.K2 = a.K2; p.alpha2 = a.alpha2;
  p.C = a.C; p.ldc = a.ldc; p.sC = a.sC;
  p.Cb = static_cast<__nv_bfloat16*>(a.C_bf16);
  p.C2 = a.C2; p.alpha_c2 = a.alpha_c2; p.diag2 = a.diag2;
  p.M = a.M; p.N = a.N; p.K = a.K; p.batch = a.batch;
  p.alpha = a.alpha;
  p.nadd = a.nadd;
  for (int q = 0; q < 8; ++q) {
    p.add[q] = a.add[q];
    p.addc[q] = a.addc[q];
    p.addc2[q] = a.addc2[q];
  }
  p.skew_add = a.skew_add;
  p.skew_c = a.skew_c;
  p.diag = a.diag;
  p.mode = a.mode;
  return p;
}

cudaError_t launch_cnp_mm(const SgemmArgs& a, cudaStream_t s) {
  SgemmDev p = make_dev(a);
  const int nt = a.M / 64;
  p.nt = nt;
  p.tiles_n = nt;
  p.tiles_per_batch = a.mode == SG_FULL ? nt * nt : nt * (nt + 1) / 2;
  const int64_t grid = (int64_t)p.tiles_per_batch * a.batch;
  if (grid > 0x7fffffff) return cudaErrorInvalidValue;
  const bool rows = a.a_sym != 0 && (!a.A2 || (a.a2_sym != 0 && (a.alpha2 == 1.f || a.alpha2 == -1.f)));
  begin_launch("cnp_sgemm", s);
  if (rows)
    k_cnp_mm<true><<<(unsigned)grid, kMMThreads, 0, s>>>(p, a.a_sym, a.a2_sym);
  else
    k_cnp_mm<false><<<(unsigned)grid, kMMThreads, 0, s>>>(p, a.a_sym, a.a2_sym);
  end_launch("cnp_sgemm", s);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sgemm(const SgemmArgs& a, cudaStream_t s) {
  if (a.batch <= 0 || a.M <= 0 || a.N <= 0) return cudaSuccess;
  // square b x b blocks with b % 64 == 0 and no transposed operand: the lean kernel
  const int bsq = a.M;
  const bool square = a.M == a.N && a.K == bsq && (!a.A2 || a.K2 == bsq) && bsq % 64 == 0 &&
                      a.lda == bsq && a.ldb == bsq && a.ldc == bsq &&
                      (!a.A2 || (a.lda2 == bsq && a.ldb2 == bsq)) && !a.transA && !a.transB &&
                      !a.transA2 && !a.transB2 && a.nadd <= 8;
  if (square) return launch_cnp_mm(a, s);
  if (a.a_sym == 2 || a.a2_sym == 2) {  // operand given as its transpose
    SgemmArgs t = a;
    if (t.a_sym == 2) { t.transA = !t.transA; t.a_sym = 0; }
    if (t.a2_sym == 2) { t.transA2 = !t.transA2; t.a2_sym = 0; }
    return launch_sgemm(t, s);
  }
  SgemmDev p;
  p.A = a.A; p.lda = a.lda; p.sA = a.sA;
  p.B = a.B; p.ldb = a.ldb; p.sB = a.sB;
  p.transA = a.transA; p.transB = a.transB;
  p.A2 = a.A2; p.lda2 = a.lda2; p.sA2 = a.sA2;
  p.B2 = a.B2; p.ldb2 = a.ldb2; p.sB2 = a.sB2;
  p.transA2 = a.transA2; p.transB2 = a.transB2;
  p.K2 = a.K2; p.alpha2 = a.alpha2;
  p.C = a.C; p.ldc = a.ldc; p.sC = a.sC;
  p.Cb = static_cast<__nv_bfloat16*>(a.C_bf16);
  p.C2 = a.C2; p.alpha_c2 = a.alpha_c2; p.diag2 = a.diag2;
  p.M = a.M; p.N = a.N; p.K = a.K; p.batch = a.batch;
  p.alpha = a.alpha;
  p.nadd = a.nadd;
  for (int q = 0; q < 8; ++q) {
    p.add[q] = a.add[q];
    p.addc[q] = a.addc[q];
    p.addc2[q] = a.addc2[q];
  }
  p.skew_add = a.skew_add;
  p.skew_c = a.skew_c;
  p.diag = a.diag;
  p.mode = a.mode;
  // tile size: 128 for large matrices, 64 / 32 for small ones
  const int big = a.M > a.N ? a.M : a.N;
  int TM = big >= 128 ? 8 : (big >= 64 ? 4 : 2);
  auto tiles_for = [&](int tm) {
    int bm = 16 * tm;
    if (a.mode == SG_FULL) return (int64_t)ceil_div(a.M, bm) * ceil_div(a.N, bm);
    int nt = ceil_div(a.M, bm);
    return (int64_t)nt * (nt + 1) / 2;
  };
  // keep enough CTAs in flight for small batches (64-wide tiles still keep FFMA:LDS high)
  if (TM == 8 && tiles_for(8) * a.batch < 2 * num_sms()) TM = 4;
  const int bm = 16 * TM;
  p.tiles_n = ceil_div(a.N, bm);
  p.nt = ceil_div(a.M, bm);
  p.tiles_per_batch = (int)tiles_for(TM);
  const int64_t grid = (int64_t)p.tiles_per_batch * a.batch;
  if (grid > 0x7fffffff) return cudaErrorInvalidValue;
  begin_launch("cnp_sgemm", s);
  if (TM == 8)
    k_sgemm<8, 16><<<(unsigned)grid, kThreads, 0, s>>>(p);
  else if (TM == 4)
    k_sgemm<4, 32><<<(unsigned)grid, kThreads, 0, s>>>(p);
  else
    k_sgemm<2, 32><<<(unsigned)grid, kThreads, 0, s>>>(p);
  end_launch("cnp_sgemm", s);
  return cudaGetLastError();
}

cudaError_t launch_theta_to_Q(const float* theta, float* Q, int nblk, int b, cudaStream_t s) {
  if (nblk <= 0) return cudaSuccess;
  const int nt = ceil_div(b, 32), pairs = nt * (nt + 1) / 2;
  begin_launch("cnp_elementwise", s);
  k_theta_to_Q<<<nblk * pairs, 256, 0, s>>>(theta, Q, b, nt, pairs);
  end_launch("cnp_elementwise", s);
  return cudaGetLastError();
}

cudaError_t launch_symcomb(const float* const* X, int nin, float* const* out, int nout,
                           const float* coef, int nblk, int b, cudaStream_t s, float* tout) {
  if (nblk <= 0) return cudaSuccess;
  if (nin < 1 || nin > 4 || nout < 1 || nout > 4) return cudaErrorInvalidValue;
  SymcombDev p;
  p.tout = tout;
  for (int i = 0; i < 4; ++i) {
    p.X[i] = i < nin ? X[i] : nullptr;
    p.out[i] = i < nout ? out[i] : nullptr;
    for (int j = 0; j < 4; ++j) p.coef[i][j] = (i < nout && j < nin) ? coef[i * nin + j] : 0.f;
  }
  p.nin = nin;
  p.nout = nout;
  const int nt = ceil_div(b, 32), pairs = nt * (nt + 1) / 2;
  begin_launch("cnp_elementwise", s);
  k_symcomb<<<nblk * pairs, 256, 0, s>>>(p, b, nt, pairs);
  end_launch("cnp_elementwise", s);
  return cudaGetLastError();
}

cudaError_t launch_pack_skew(const float* A, float* dtheta, int nblk, int b, cudaStream_t s) {
  if (nblk <= 0) return cudaSuccess;
  const int nt = ceil_div(b, 32), pairs = nt * (nt + 1) / 2;
  begin_launch("cnp_elementwise", s);
  k_pack_skew<<<nblk * pairs, 256, 0, s>>>(A, dtheta, b, nt, pairs);
  end_launch("cnp_elementwise", s);
  return cudaGetLastError();
}

cudaError_t launch_split_reduce(const float* src, int nsplit, int64_t stride, float* dst,
                                int64_t count, int accumulate, cudaStream_t s) {
  if (count <= 0) return cudaSuccess;
  int64_t blocks = (count / 4 + 255) / 256;
  if (blocks < 1) blocks = 1;
  if (blocks > num_sms() * 8) blocks = num_sms() * 8;
  begin_launch("reduce", s);
  const cudaError_t e = launch_pdl(k_split_reduce, dim3((unsigned)blocks), dim3(256), 0, s, src,
                                   nsplit, stride, dst, count, accumulate);
  end_launch("reduce", s);
  return e;
}

cudaError_t launch_f32_to_bf16(const float* src, void* dst, int64_t count, cudaStream_t s) {
  if (count <= 0) return cudaSuccess;
  int64_t blocks = (count + 255) / 256;
  if (blocks > num_sms() * 8) blocks = num_sms() * 8;
  begin_launch("convert", s);
  k_f32_to_bf16<<<(unsigned)blocks, 256, 0, s>>>(src, static_cast<__nv_bfloat16*>(dst), count);
  end_launch("convert", s);
  return cudaGetLastError();
}

}  // namespace poetx
