// The Cayley-Neumann parameterisation for small blocks (b = 32 or 64) with every matrix of a
// block in shared memory: one launch per call, no device scratch (POET-X technical summary
// section 2.4: the fused CNP kernel keeps Q and its powers on chip and fuses the Neumann
// sum).
//
// Notation: Q = skew(theta), S = Q^2, d = floor((k + 1) / 2), c_i = 1 for i = 0 and k + 1 and
// 2 otherwise, e_j = c_2j, f_j = c_2j+1,  G = E(S) + Q F(S) = E + f_0 Q + Q F' with
// E = sum_j e_j S^j and F' = sum_{j>=1} f_j S^j.
//
// Forward, per block: Q from theta; S = Q Q; P_j = S P_{j-1} (j = 2..d) while E and F' are
// summed in registers; G = E + f_0 Q + Q F'.
//
// Backward, per block, with dG the gradient of G: D = Q dG; N_j = e_j (dG + dG^T) -
// f_j (D + D^T) (the upstream of S^j, symmetric); the adjoint of S,
//   Y = sum_{j=1..d} sum_{a=0..j-1} S^a N_j S^(j-1-a),
// by the two-sided recursion U_d = R_d = N_d, R_l = N_l + R_{l+1} S,
// U_l = N_l + S U_{l+1} + R_{l+1} S, Y = U_1; then A = f_0 dG + dG F' - Y Q and
// dtheta_(i,j) = A_ij - A_ji (i < j).  Q, S and F' come from the forward's saved copies or
// are recomputed.
//
// Layout: each matrix is B rows of B + 4 floats in shared memory.  A block's B x B outputs
// are split over (B / 4)^2 threads, 4 x 4 each (rows 4 ty.., columns 4 tx..); a CTA of 256
// threads holds 256 / (B / 4)^2 blocks (1 for b = 64, 4 for b = 32).  Every product reads A
// through its transpose (At, row k = column k of A): the symmetric and skew operands are
// their own transposes up to sign, and the general ones are kept transposed.  Per k step a
// thread issues two 16-byte shared loads and 16 FMAs (as 8 packed pairs).
#include <cuda_bf16.h>

#include "poetx_internal.h"

namespace poetx {
namespace {

constexpr int kFzThreads = 256;
constexpr int kFzFwdMats = 4;  // Q, S, F', one work matrix
constexpr int kFzBwdMats = 6;  // Q, S, F', dG, U, R^T

template <int B>
struct Fz {
  static constexpr int LD = B + 4;               // padded row (floats), 16-byte aligned
  static constexpr int MAT = B * LD;             // floats per matrix
  static constexpr int TPB = (B / 4) * (B / 4);  // threads per block
  static constexpr int BPC = kFzThreads / TPB;   // blocks per CTA
};

struct FzCoef {
  int d;
  float e[10], f[10];
};

__device__ __forceinline__ int64_t tri_index(int i, int j, int b) {
  // strict upper triangle, row-major: (i, j), i < j
  return (int64_t)i * b - (int64_t)i * (i + 1) / 2 + (j - i - 1);
}

#ifndef FZ_FMA2
#define FZ_FMA2 1
#endif

// acc = A Bm with At = A^T (row k of At = column k of A); acc is overwritten.
// With FZ_FMA2 the 16 FMAs of a k step run as 8 packed pairs (fma.rn.f32x2: two fp32 fused
// multiply-adds, each rounded once as fmaf, in the same order over k), on the pairs
//   D[p][q] = (acc[2p][2q],     acc[2p + 1][2q + 1]) += (a[2p], a[2p + 1]) * (b[2q], b[2q + 1])
//   X[p][q] = (acc[2p][2q + 1], acc[2p + 1][2q])     += (a[2p], a[2p + 1]) * (b[2q + 1], b[2q])
// whose a and b pairs are halves of the 16-byte loads.
template <int B>
__device__ __forceinline__ void fz_mm(const float* __restrict__ At, const float* __restrict__ Bm,
                                      int tx, int ty, float (&acc)[4][4]) {
  constexpr int LD = Fz<B>::LD;
#if FZ_FMA2
  unsigned long long D[2][2] = {{0ull, 0ull}, {0ull, 0ull}};  // (+0.f, +0.f)
  unsigned long long X[2][2] = {{0ull, 0ull}, {0ull, 0ull}};
#pragma unroll 8
  for (int k = 0; k < B; ++k) {
    const ulonglong2 a = *reinterpret_cast<const ulonglong2*>(At + k * LD + 4 * ty);
    const ulonglong2 b = *reinterpret_cast<const ulonglong2*>(Bm + k * LD + 4 * tx);
    const unsigned long long ap[2] = {a.x, a.y}, bp[2] = {b.x, b.y};
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      unsigned long long bs;  // (b[2q + 1], b[2q])
      asm("{\n\t.reg .b32 lo, hi;\n\tmov.b64 {lo, hi}, %1;\n\tmov.b64 %0, {hi, lo};\n\t}"
          : "=l"(bs) : "l"(bp[q]));
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(D[p][q]) : "l"(ap[p]), "l"(bp[q]));
        asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(X[p][q]) : "l"(ap[p]), "l"(bs));
      }
    }
  }
#pragma unroll
  for (int p = 0; p < 2; ++p)
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      asm("mov.b64 {%0, %1}, %2;" : "=f"(acc[2 * p][2 * q]), "=f"(acc[2 * p + 1][2 * q + 1])
          : "l"(D[p][q]));
      asm("mov.b64 {%0, %1}, %2;" : "=f"(acc[2 * p][2 * q + 1]), "=f"(acc[2 * p + 1][2 * q])
          : "l"(X[p][q]));
    }
#else
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;
#pragma unroll 8
  for (int k = 0; k < B; ++k) {
    const float4 a = *reinterpret_cast<const float4*>(At + k * LD + 4 * ty);
    const float4 b = *reinterpret_cast<const float4*>(Bm + k * LD + 4 * tx);
    const float av[4] = {a.x, a.y, a.z, a.w};
    const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(av[r], bv[c], acc[r][c]);
  }
#endif
}

template <int B>
__device__ __forceinline__ void fz_store(float* M, int tx, int ty, const float (&v)[4][4]) {
  constexpr int LD = Fz<B>::LD;
#pragma unroll
  for (int r = 0; r < 4; ++r)
    *reinterpret_cast<float4*>(M + (4 * ty + r) * LD + 4 * tx) =
        make_float4(v[r][0], v[r][1], v[r][2], v[r][3]);
}
// stores v^T: element (i, j) of the thread's block goes to (j, i)
template <int B>
__device__ __forceinline__ void fz_store_t(float* M, int tx, int ty, const float (&v)[4][4]) {
  constexpr int LD = Fz<B>::LD;
#pragma unroll
  for (int c = 0; c < 4; ++c)
    *reinterpret_cast<float4*>(M + (4 * tx + c) * LD + 4 * ty) =
        make_float4(v[0][c], v[1][c], v[2][c], v[3][c]);
}
template <int B>
__device__ __forceinline__ void fz_load(const float* M, int tx, int ty, float (&v)[4][4]) {
  constexpr int LD = Fz<B>::LD;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const float4 x = *reinterpret_cast<const float4*>(M + (4 * ty + r) * LD + 4 * tx);
    v[r][0] = x.x; v[r][1] = x.y; v[r][2] = x.z; v[r][3] = x.w;
  }
}
// the thread's 4 x 4 block of M^T
template <int B>
__device__ __forceinline__ void fz_load_t(const float* M, int tx, int ty, float (&v)[4][4]) {
  constexpr int LD = Fz<B>::LD;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const float4 x = *reinterpret_cast<const float4*>(M + (4 * tx + c) * LD + 4 * ty);
    v[0][c] = x.x; v[1][c] = x.y; v[2][c] = x.z; v[3][c] = x.w;
  }
}

// global b x b fp32 block <-> shared matrix (the thread's 4 x 4 block, 16-byte accesses)
template <int B>
__device__ __forceinline__ void fz_from_global(float* M, const float* __restrict__ g, int tx,
                                               int ty) {
  constexpr int LD = Fz<B>::LD;
#pragma unroll
  for (int r = 0; r < 4; ++r)
    *reinterpret_cast<float4*>(M + (4 * ty + r) * LD + 4 * tx) =
        __ldg(reinterpret_cast<const float4*>(g + (int64_t)(4 * ty + r) * B + 4 * tx));
}
template <int B>
__device__ __forceinline__ void fz_to_global(float* __restrict__ g, int tx, int ty,
                                             const float (&v)[4][4]) {
#pragma unroll
  for (int r = 0; r < 4; ++r)
    __stcg(reinterpret_cast<float4*>(g + (int64_t)(4 * ty + r) * B + 4 * tx),
           make_float4(v[r][0], v[r][1], v[r][2], v[r][3]));
}

// Q = skew(theta) into shared memory
template <int B>
__device__ __forceinline__ void fz_expand(float* Qs, const float* __restrict__ th, int tx, int ty) {
  float q[4][4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int i = 4 * ty + r, j = 4 * tx + c;
      q[r][c] = i < j ? __ldg(th + tri_index(i, j, B))
                      : (i > j ? -__ldg(th + tri_index(j, i, B)) : 0.f);
    }
  fz_store<B>(Qs, tx, ty, q);
}

// S = Q Q and F' = sum_{j>=1} f_j S^j into shared memory (Ss, Fs), with E = e_0 I +
// sum_{j>=1} e_j S^j returned in registers when want_e.  W: work matrix (the powers S^j,
// j >= 2, one after another: each is written only after every thread has read the last).
template <int B>
__device__ __forceinline__ void fz_powers(const float* Qs, float* Ss, float* Fs, float* W,
                                          const FzCoef& P, int tx, int ty, float (&E)[4][4],
                                          bool want_e) {
  float acc[4][4], F[4][4];
  fz_mm<B>(Qs, Qs, tx, ty, acc);  // rows of Q = columns of Q^T = -columns of Q
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[r][c] = -acc[r][c];
  fz_store<B>(Ss, tx, ty, acc);
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const bool diag = 4 * ty + r == 4 * tx + c;
      E[r][c] = (diag ? P.e[0] : 0.f) + P.e[1] * acc[r][c];
      F[r][c] = P.f[1] * acc[r][c];
    }
  const float* prev = Ss;
  for (int j = 2; j <= P.d; ++j) {
    __syncthreads();  // P_{j-1} is complete
    fz_mm<B>(Ss, prev, tx, ty, acc);  // S is symmetric: its rows are its columns
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (want_e) E[r][c] = fmaf(P.e[j], acc[r][c], E[r][c]);
        F[r][c] = fmaf(P.f[j], acc[r][c], F[r][c]);
      }
    if (j < P.d) {
      if (prev == W) __syncthreads();  // every thread has read S^(j-1) from W
      fz_store<B>(W, tx, ty, acc);
      prev = W;
    }
  }
  fz_store<B>(Fs, tx, ty, F);
}

template <int B>
__global__ void __launch_bounds__(kFzThreads)
    k_cnp_fused_fwd(const float* __restrict__ theta, float* __restrict__ G,
                    __nv_bfloat16* __restrict__ Gb, float* __restrict__ Qo,
                    float* __restrict__ So, float* __restrict__ Fo, int nblk, const FzCoef P) {
  using C = Fz<B>;
  extern __shared__ __align__(16) float fz_smem[];
  const int sb = threadIdx.x / C::TPB, t = threadIdx.x % C::TPB;
  const int tx = t % (B / 4), ty = t / (B / 4);
  float* base = fz_smem + sb * kFzFwdMats * C::MAT;
  float *Qs = base, *Ss = base + C::MAT, *Fs = base + 2 * C::MAT, *W = base + 3 * C::MAT;
  const int64_t blk = (int64_t)blockIdx.x * C::BPC + sb;
  const bool live = blk < nblk;  // (every thread still meets every barrier)
  const int64_t bb = (int64_t)B * B;
  pdl_trigger();
  pdl_wait();
  if (live) fz_expand<B>(Qs, theta + blk * ((int64_t)B * (B - 1) / 2), tx, ty);
  __syncthreads();
  float E[4][4];
  fz_powers<B>(Qs, Ss, Fs, W, P, tx, ty, E, true);
  __syncthreads();  // F' is complete
  float acc[4][4], q[4][4];
  fz_mm<B>(Qs, Fs, tx, ty, acc);  // -(Q F')
  fz_load<B>(Qs, tx, ty, q);
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[r][c] = E[r][c] + P.f[0] * q[r][c] - acc[r][c];
  if (!live) return;
  fz_to_global<B>(G + blk * bb, tx, ty, acc);
  if (Gb) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      __nv_bfloat162 lo = __floats2bfloat162_rn(acc[r][0], acc[r][1]);
      __nv_bfloat162 hi = __floats2bfloat162_rn(acc[r][2], acc[r][3]);
      uint2 u;
      u.x = *reinterpret_cast<uint32_t*>(&lo);
      u.y = *reinterpret_cast<uint32_t*>(&hi);
      __stcg(reinterpret_cast<uint2*>(Gb + blk * bb + (int64_t)(4 * ty + r) * B + 4 * tx), u);
    }
  }
  if (Qo) {
    float v[4][4];
    fz_to_global<B>(Qo + blk * bb, tx, ty, q);
    fz_load<B>(Ss, tx, ty, v);
    fz_to_global<B>(So + blk * bb, tx, ty, v);
    fz_load<B>(Fs, tx, ty, v);
    fz_to_global<B>(Fo + blk * bb, tx, ty, v);
  }
}

template <int B>
__global__ void __launch_bounds__(kFzThreads)
    k_cnp_fused_bwd(const float* __restrict__ theta, const float* __restrict__ dG,
                    const float* __restrict__ Qi, const float* __restrict__ Si,
                    const float* __restrict__ Fi, float* __restrict__ dtheta, int nblk,
                    const FzCoef P) {
  using C = Fz<B>;
  extern __shared__ __align__(16) float fz_smem[];
  const int sb = threadIdx.x / C::TPB, t = threadIdx.x % C::TPB;
  const int tx = t % (B / 4), ty = t / (B / 4);
  float* base = fz_smem + sb * kFzBwdMats * C::MAT;
  // Q, S, F', dG, and U and R^T of the recursion (single buffers: each level reads them all
  // before any thread writes the next level)
  float *Qs = base, *Ss = base + C::MAT, *Fs = base + 2 * C::MAT, *Gs = base + 3 * C::MAT,
        *Us = base + 4 * C::MAT, *Rs = base + 5 * C::MAT;
  const int64_t blk = (int64_t)blockIdx.x * C::BPC + sb;
  const bool live = blk < nblk;
  const int64_t bb = (int64_t)B * B, ntri = (int64_t)B * (B - 1) / 2;
  pdl_trigger();
  pdl_wait();
  float acc[4][4], acc2[4][4], v[4][4];
  if (live) {
    fz_from_global<B>(Gs, dG + blk * bb, tx, ty);
    if (Si) {
      fz_from_global<B>(Qs, Qi + blk * bb, tx, ty);
      fz_from_global<B>(Ss, Si + blk * bb, tx, ty);
      fz_from_global<B>(Fs, Fi + blk * bb, tx, ty);
    } else {
      fz_expand<B>(Qs, theta + blk * ntri, tx, ty);
    }
  }
  __syncthreads();
  if (!Si) {  // the forward's S and F' again (U as work space)
    float E[4][4];
    fz_powers<B>(Qs, Ss, Fs, Us, P, tx, ty, E, false);
    __syncthreads();
  }
  // X1 = dG + dG^T, and D = Q dG = -(rows of Q) dG
  float x1[4][4], x2[4][4];
  {
    float g[4][4], gt[4][4];
    fz_load<B>(Gs, tx, ty, g);
    fz_load_t<B>(Gs, tx, ty, gt);
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) x1[r][c] = g[r][c] + gt[r][c];
  }
  fz_mm<B>(Qs, Gs, tx, ty, acc);
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[r][c] = -acc[r][c];
  fz_store<B>(Us, tx, ty, acc);  // D (temporarily)
  __syncthreads();
  // X2 = D + D^T;  N_j = e_j X1 - f_j X2
  fz_load_t<B>(Us, tx, ty, v);
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) x2[r][c] = acc[r][c] + v[r][c];
  __syncthreads();  // D is no longer read
  // U_d = R_d = N_d
  const int d = P.d;
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) v[r][c] = P.e[d] * x1[r][c] - P.f[d] * x2[r][c];
  fz_store<B>(Us, tx, ty, v);
  fz_store_t<B>(Rs, tx, ty, v);
  for (int l = d - 1; l >= 1; --l) {
    __syncthreads();  // U_{l+1}, R_{l+1} are complete
    fz_mm<B>(Ss, Us, tx, ty, acc);   // S U_{l+1}
    fz_mm<B>(Rs, Ss, tx, ty, acc2);  // R_{l+1} S
    float u[4][4], rr[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float n = P.e[l] * x1[r][c] - P.f[l] * x2[r][c];
        rr[r][c] = n + acc2[r][c];
        u[r][c] = rr[r][c] + acc[r][c];
      }
    __syncthreads();  // every thread has read U_{l+1} and R_{l+1}
    fz_store<B>(Us, tx, ty, u);
    fz_store_t<B>(Rs, tx, ty, rr);
  }
  __syncthreads();  // Y = U_1 is complete; R is no longer read
  // dG^T into R's buffer, then A = f_0 dG + dG F' - Y Q  (Y symmetric)
  fz_load<B>(Gs, tx, ty, v);
  fz_store_t<B>(Rs, tx, ty, v);
  __syncthreads();
  fz_mm<B>(Rs, Fs, tx, ty, acc);
  fz_mm<B>(Us, Qs, tx, ty, acc2);
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) v[r][c] = P.f[0] * v[r][c] + acc[r][c] - acc2[r][c];
  fz_store<B>(Ss, tx, ty, v);  // A (S is no longer read)
  __syncthreads();
  if (!live) return;
  float at[4][4];
  fz_load_t<B>(Ss, tx, ty, at);
  float* th = dtheta + blk * ntri;
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int i = 4 * ty + r, j = 4 * tx + c;
      if (i < j) th[tri_index(i, j, B)] = v[r][c] - at[r][c];
    }
}

FzCoef fz_coef(int k) {
  FzCoef p;
  p.d = (k + 1) / 2;
  for (int j = 0; j < 10; ++j) {
    auto c = [&](int i) -> float {
      if (i < 0 || i > k + 1) return 0.f;
      return (i == 0 || i == k + 1) ? 1.f : 2.f;
    };
    p.e[j] = c(2 * j);
    p.f[j] = c(2 * j + 1);
  }
  return p;
}

// (one instantiation, and so one flag set, per kernel: B and direction)
template <int B, bool FWD, typename K>
cudaError_t fz_attr(K kern, size_t smem) {
  static bool done[64] = {false};  // once per device, outside any stream capture
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (done[dev]) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess) done[dev] = true;
  return e;
}

template <int B>
cudaError_t fwd_t(const float* theta, float* G, void* Gb, float* Qo, float* So, float* Fo,
                  int nblk, int k, cudaStream_t s) {
  using C = Fz<B>;
  const size_t smem = (size_t)C::BPC * kFzFwdMats * C::MAT * sizeof(float);
  cudaError_t e = fz_attr<B, true>(k_cnp_fused_fwd<B>, smem);
  if (e != cudaSuccess) return e;
  const int grid = (nblk + C::BPC - 1) / C::BPC;
  begin_launch("cnp_sgemm", s);
  e = launch_pdl(k_cnp_fused_fwd<B>, dim3(grid), dim3(kFzThreads), smem, s, theta, G,
                 static_cast<__nv_bfloat16*>(Gb), Qo, So, Fo, nblk, fz_coef(k));
  end_launch("cnp_sgemm", s);
  return e;
}

template <int B>
cudaError_t bwd_t(const float* theta, const float* dG, const float* Qi, const float* Si,
                  const float* Fi, float* dtheta, int nblk, int k, cudaStream_t s) {
  using C = Fz<B>;
  const size_t smem = (size_t)C::BPC * kFzBwdMats * C::MAT * sizeof(float);
  cudaError_t e = fz_attr<B, false>(k_cnp_fused_bwd<B>, smem);
  if (e != cudaSuccess) return e;
  const int grid = (nblk + C::BPC - 1) / C::BPC;
  begin_launch("cnp_sgemm", s);
  e = launch_pdl(k_cnp_fused_bwd<B>, dim3(grid), dim3(kFzThreads), smem, s, theta, dG, Qi, Si,
                 Fi, dtheta, nblk, fz_coef(k));
  end_launch("cnp_sgemm", s);
  return e;
}

}  // namespace

bool cnp_fused_ok(int b, int k) { return (b == 32 || b == 64) && k >= 1 && k <= 16; }

cudaError_t launch_cnp_fused_fwd(const float* theta, float* G, void* G_bf16, float* Q_save,
                                 float* S_save, float* F_save, int nblk, int b, int k,
                                 cudaStream_t s) {
  if (nblk <= 0) return cudaSuccess;
  if (!cnp_fused_ok(b, k) || ((Q_save != nullptr) != (S_save != nullptr)) ||
      ((Q_save != nullptr) != (F_save != nullptr)))
    return cudaErrorInvalidValue;
  return b == 64 ? fwd_t<64>(theta, G, G_bf16, Q_save, S_save, F_save, nblk, k, s)
                 : fwd_t<32>(theta, G, G_bf16, Q_save, S_save, F_save, nblk, k, s);
}

cudaError_t launch_cnp_fused_bwd(const float* theta, const float* dG, const float* Q_saved,
                                 const float* S_saved, const float* F_saved, float* dtheta,
                                 int nblk, int b, int k, cudaStream_t s) {
  if (nblk <= 0) return cudaSuccess;
  if (!cnp_fused_ok(b, k) || ((Q_saved != nullptr) != (S_saved != nullptr)) ||
      ((Q_saved != nullptr) != (F_saved != nullptr)))
    return cudaErrorInvalidValue;
  return b == 64 ? bwd_t<64>(theta, dG, Q_saved, S_saved, F_saved, dtheta, nblk, k, s)
                 : bwd_t<32>(theta, dG, Q_saved, S_saved, F_saved, dtheta, nblk, k, s);
}

}  // namespace poetx
