// fp32 SIMT kernels: a batched FFMA GEMM with structured (symmetric / symmetric+skew)
// outputs, and the small elementwise kernels of the Cayley-Neumann parameterisation
// (POET-X technical summary, section 2.4).
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
constexpr int kBK = 16;

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
template <int TM>
struct Tile {
  static constexpr int VEC = TM < 4 ? TM : 4;
  static constexpr int NG = TM / VEC;
  static constexpr int BM = 16 * TM;
  static constexpr int LOADS = BM * kBK / kThreads;  // elements per thread per operand tile
};

template <int TM>
__device__ __forceinline__ void load_tile_regs(float (&r)[Tile<TM>::LOADS], const float* X,
                                               int64_t ldx, int trans, int row0, int k0,
                                               int rows, int kdim, float scale, bool is_b) {
  // Loads the (BM x kBK) tile of op(X) (for A) or the (kBK x BN) tile of op(B), as
  // element (row, k) with row in [row0, row0+BM), k in [k0, k0+kBK).
  // A: op(A)[i][k] = trans ? X[k*ld + i] : X[i*ld + k]
  // B: op(B)[k][j] = trans ? X[j*ld + k] : X[k*ld + j]   (j plays the role of row)
  constexpr int BM = Tile<TM>::BM;
  const int tid = threadIdx.x;
  const bool k_contig = is_b ? (trans != 0) : (trans == 0);
#pragma unroll
  for (int l = 0; l < Tile<TM>::LOADS; ++l) {
    int idx = tid + l * kThreads;
    int i, k;
    if (k_contig) {
      i = idx / kBK;
      k = idx % kBK;
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

template <int TM>
__device__ __forceinline__ void store_tile_smem(const float (&r)[Tile<TM>::LOADS],
                                                float (*S)[Tile<TM>::BM + 4], int trans,
                                                bool is_b) {
  constexpr int BM = Tile<TM>::BM;
  const int tid = threadIdx.x;
  const bool k_contig = is_b ? (trans != 0) : (trans == 0);
#pragma unroll
  for (int l = 0; l < Tile<TM>::LOADS; ++l) {
    int idx = tid + l * kThreads;
    int i, k;
    if (k_contig) {
      i = idx / kBK;
      k = idx % kBK;
    } else {
      k = idx / BM;
      i = idx % BM;
    }
    S[k][i] = r[l];
  }
}

template <int TM>
__global__ void __launch_bounds__(kThreads) k_sgemm(SgemmDev p) {
  using TL = Tile<TM>;
  constexpr int BM = TL::BM, VEC = TL::VEC, NG = TL::NG;
  __shared__ __align__(16) float As[2][kBK][BM + 4];
  __shared__ __align__(16) float Bs[2][kBK][BM + 4];

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
  const int nk1 = (p.K + kBK - 1) / kBK;
  const int nk2 = p.A2 ? (p.K2 + kBK - 1) / kBK : 0;
  const int nkt = nk1 + nk2;

  auto load = [&](int kt) {
    if (kt < nk1) {
      load_tile_regs<TM>(ra, p.A + bz * p.sA, p.lda, p.transA, m0, kt * kBK, p.M, p.K, 1.f,
                         false);
      load_tile_regs<TM>(rb, p.B + bz * p.sB, p.ldb, p.transB, n0, kt * kBK, p.N, p.K, 1.f, true);
    } else {
      int k2 = (kt - nk1) * kBK;
      load_tile_regs<TM>(ra, p.A2 + bz * p.sA2, p.lda2, p.transA2, m0, k2, p.M, p.K2, p.alpha2,
                         false);
      load_tile_regs<TM>(rb, p.B2 + bz * p.sB2, p.ldb2, p.transB2, n0, k2, p.N, p.K2, 1.f, true);
    }
  };
  auto store = [&](int kt, int buf) {
    int ta = kt < nk1 ? p.transA : p.transA2;
    int tb = kt < nk1 ? p.transB : p.transB2;
    store_tile_smem<TM>(ra, As[buf], ta, false);
    store_tile_smem<TM>(rb, Bs[buf], tb, true);
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
    for (int k = 0; k < kBK; ++k) {
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
#pragma unroll
  for (int gi = 0; gi < NG; ++gi)
#pragma unroll
    for (int vi = 0; vi < VEC; ++vi) {
      const int i = m0 + gi * 16 * VEC + ty * VEC + vi;
      if (i >= p.M) continue;
#pragma unroll
      for (int gj = 0; gj < NG; ++gj)
#pragma unroll
        for (int vj = 0; vj < VEC; ++vj) {
          const int j = n0 + gj * 16 * VEC + tx * VEC + vj;
          if (j >= p.N) continue;
          if (p.mode != SG_FULL && I == J && i > j) continue;  // mirror of (j, i)
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
          const int64_t ji = (int64_t)j * p.ldc + i;
          if (p.mode == SG_SYMSKEW) {
            if (i == j) {
              C[ij] = sym;
              if (Cb) Cb[ij] = __float2bfloat16_rn(sym);
            } else {
              C[ij] = sym + skew;
              C[ji] = sym - skew;
              if (Cb) {
                Cb[ij] = __float2bfloat16_rn(sym + skew);
                Cb[ji] = __float2bfloat16_rn(sym - skew);
              }
            }
          } else {
            const float v = skew + sym;
            C[ij] = v;
            if (Cb) Cb[ij] = __float2bfloat16_rn(v);
            const float v2 = p.alpha_c2 * a + sym2;
            if (C2) C2[ij] = v2;
            if (p.mode == SG_SYM && i != j) {
              C[ji] = v;
              if (Cb) Cb[ji] = __float2bfloat16_rn(v);
              if (C2) C2[ji] = v2;
            }
          }
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
  const int64_t n4 = count / 4;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    float4 acc = accumulate ? reinterpret_cast<const float4*>(dst)[i] : make_float4(0, 0, 0, 0);
    for (int s = 0; s < nsplit; ++s) {
      float4 v = __ldg(reinterpret_cast<const float4*>(src + s * stride) + i);
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
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

}  // namespace

cudaError_t launch_sgemm(const SgemmArgs& a, cudaStream_t s) {
  if (a.batch <= 0 || a.M <= 0 || a.N <= 0) return cudaSuccess;
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
    k_sgemm<8><<<(unsigned)grid, kThreads, 0, s>>>(p);
  else if (TM == 4)
    k_sgemm<4><<<(unsigned)grid, kThreads, 0, s>>>(p);
  else
    k_sgemm<2><<<(unsigned)grid, kThreads, 0, s>>>(p);
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
                           const float* coef, int nblk, int b, cudaStream_t s) {
  if (nblk <= 0) return cudaSuccess;
  if (nin < 1 || nin > 4 || nout < 1 || nout > 4) return cudaErrorInvalidValue;
  SymcombDev p;
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
  k_split_reduce<<<(unsigned)blocks, 256, 0, s>>>(src, nsplit, stride, dst, count, accumulate);
  end_launch("reduce", s);
  return cudaGetLastError();
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
