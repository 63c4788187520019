// Internal declarations shared by the libpoetx translation units (host side).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <string>
#include <utility>

#include "../../include/poetx.h"

namespace poetx {

// ---- error reporting -------------------------------------------------------------
void set_error(const std::string& msg);
int fail(int status, const std::string& msg);
int cuda_fail(cudaError_t e, const char* what);

// Launch accounting: every kernel launch goes through begin_launch/end_launch, which
// count it and, when the profiler watches that kernel family, bracket it with events.
void begin_launch(const char* family, cudaStream_t s);
void end_launch(const char* family, cudaStream_t s);

// Device error flag (set by kernels whose bounded waits time out).  nullptr when the flag's
// device address cannot be looked up; launchers then refuse to launch.
int* device_error_flag();

// Time limit of every bounded wait in the kernels, in nanoseconds (poetx_set_wait_limit).
unsigned long long wait_limit_ns();

// Number of SMs of the current device.
int num_sms();

// CNP forward scratch: bytes per block (its matrices and task-graph counters) and the
// fixed part of a call (the chunking of poetx_cnp_fwd works in these units).
size_t cnp_fwd_block_bytes(int b, int k);
size_t cnp_fixed_bytes();

// ---- programmatic dependent launch ------------------------------------------------
// Kernels of the layer step are launched so that a kernel may start (and do its set-up)
// while the previous kernel on the stream is still finishing.  Every kernel launched this
// way calls pdl_wait() before its first access to global memory: that waits until the
// previous kernel has completed and its writes are visible, so stream order is kept.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}
#ifdef __CUDACC__
// lets the next kernel on the stream be scheduled once every CTA of this one got here
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// waits until the previous kernel on the stream has completed (its writes visible)
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
#endif

// ---- permutation / gather kernels (kernels_perm.cu) ------------------------------
// out[r, c] = in[row_idx ? row_idx[r] : r, col_idx[c]]
cudaError_t launch_gather(const void* in, void* out, const int32_t* row_idx,
                          const int32_t* col_idx, int rows, int cols, int64_t ld_in,
                          int64_t ld_out, int elem_bytes, cudaStream_t s);
// out[i] = outer[inner[i]] for i < n (composition of two index maps; indices clamped)
cudaError_t launch_compose_perm(const int32_t* outer, const int32_t* inner, int32_t* out, int n,
                                cudaStream_t s);

// ---- int8 base weight (kernels_quant.cu) -----------------------------------------
// per-row symmetric int8: s_i = max|w_i.| / 127, q = rint(w / s) in [-127, 127]
cudaError_t launch_quantize_rows(const void* W, int8_t* q, float* s, int m, int n,
                                 int elem_bytes, cudaStream_t st);
// q, s = per-row int8 codes of the merged weight W0[perm_R][:, perm_P] (no merged copy)
cudaError_t launch_merge_quantize(const void* W0, const int32_t* perm_R, const int32_t* perm_P,
                                  int8_t* q, float* s, int m, int n, int elem_bytes,
                                  cudaStream_t st);
// out (bf16) = s_i * q_ij
cudaError_t launch_dequant_rows(const int8_t* q, const float* s, void* out, int m, int n,
                                cudaStream_t st);
// out[r][c] (bf16, row stride ldo) = s_r * q[r][c] (row stride ldq) for r < rows, c < cols;
// cols % 16 == 0, 16-byte aligned rows
cudaError_t launch_dequant_2d(const int8_t* q, int64_t ldq, const float* s, void* out,
                              int64_t ldo, int rows, int cols, cudaStream_t st);

// ---- fp32 SIMT batched GEMM (kernels_sgemm.cu) -----------------------------------
enum SgemmMode { SG_FULL = 0, SG_SYM = 1, SG_SYMSKEW = 2 };

struct SgemmArgs {
  // acc = op(A) op(B) + alpha2 * op(A2) op(B2)
  // sym  = diag * delta_ij + sum_t addc[t] * add[t][i, j]
  // skew = alpha * acc + skew_c * skew_add[i, j]
  // FULL / SYM:  C = skew + sym (SYM: upper tiles computed, C_ji = C_ij)
  // SYMSKEW:     C_ij = sym + skew, C_ji = sym - skew, C_ii = sym (upper tiles computed)
  // C2 (optional, FULL / SYM only) = alpha_c2 * acc + diag2 * delta + sum addc2[t] add[t]
  const float* A = nullptr;
  int64_t lda = 0, sA = 0;
  const float* B = nullptr;
  int64_t ldb = 0, sB = 0;
  int transA = 0, transB = 0;
  const float* A2 = nullptr;
  int64_t lda2 = 0, sA2 = 0;
  const float* B2 = nullptr;
  int64_t ldb2 = 0, sB2 = 0;
  int transA2 = 0, transB2 = 0;
  int K2 = 0;
  float alpha2 = 1.f;
  float* C = nullptr;
  int64_t ldc = 0, sC = 0;  // also the layout of add[], skew_add and C2
  void* C_bf16 = nullptr;   // optional bf16 copy of C
  float* C2 = nullptr;
  float alpha_c2 = 0.f, diag2 = 0.f;
  float addc2[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  int M = 0, N = 0, K = 0, batch = 0;
  float alpha = 1.f;
  int nadd = 0;
  const float* add[8] = {nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
  float addc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const float* skew_add = nullptr;
  float skew_c = 0.f;
  float diag = 0.f;
  int mode = SG_FULL;
  // how A and A2 may be read by rows as their own transpose: 0 general, +1 symmetric,
  // -1 skew-symmetric, 2 the pointer holds the operand's transpose
  int a_sym = 0, a2_sym = 0;
};
cudaError_t launch_sgemm(const SgemmArgs& a, cudaStream_t s);

// ---- CNP elementwise kernels (kernels_sgemm.cu) -----------------------------------
// Q = skew(theta) for nblk blocks of size b.
cudaError_t launch_theta_to_Q(const float* theta, float* Q, int nblk, int b, cudaStream_t s);
// out_o = sum_s coef[o][s] * (X_s + X_s^T) for o < nout (symmetric outputs), s < nin.
// When tout is given it also receives X[0]^T.
cudaError_t launch_symcomb(const float* const* X, int nin, float* const* out, int nout,
                           const float* coef /* [nout][nin] row-major */, int nblk, int b,
                           cudaStream_t s, float* tout = nullptr);
// dtheta_idx(i,j) = A_ij - A_ji for i < j.
cudaError_t launch_pack_skew(const float* A, float* dtheta, int nblk, int b, cudaStream_t s);
// dst[j] = (accumulate ? dst[j] : 0) + sum_s src[s * stride + j], s < nsplit (fixed order).
cudaError_t launch_split_reduce(const float* src, int nsplit, int64_t stride, float* dst,
                                int64_t count, int accumulate, cudaStream_t s);
// fp32 -> bf16 (round to nearest even)
cudaError_t launch_f32_to_bf16(const float* src, void* dst, int64_t count, cudaStream_t s);

// ---- CNP for b = 32 or 64, every block's matrices in shared memory (kernels_cnp_fused.cu)
bool cnp_fused_ok(int b, int k);
// G (fp32, and its bf16 copy when G_bf16 is given) from theta; Q_save / S_save / F_save
// (all or none) receive Q, S = Q^2 and F'.  No device scratch.
cudaError_t launch_cnp_fused_fwd(const float* theta, float* G, void* G_bf16, float* Q_save,
                                 float* S_save, float* F_save, int nblk, int b, int k,
                                 cudaStream_t s);
// dtheta from dG; Q, S, F' read from the *_saved buffers (all or none) or recomputed.
cudaError_t launch_cnp_fused_bwd(const float* theta, const float* dG, const float* Q_saved,
                                 const float* S_saved, const float* F_saved, float* dtheta,
                                 int nblk, int b, int k, cudaStream_t s);

// ---- CNP as one persistent task-graph launch (kernels_cnp_graph.cu) -----------------
// Each job is one step applied to every block of a chunk; an item is one output tile of
// one job for one block.  Square blocks with b % 64 == 0; products read every A operand
// by rows (a_sym: -1 skew, +1 symmetric, 2 given as its transpose).
enum CnpJobType { JOB_EXPAND = 0, JOB_PRODUCT = 1, JOB_SYMCOMB = 2, JOB_PACK = 3 };
constexpr int kCnpMaxJobs = 14;

struct CnpJob {
  int type = JOB_PRODUCT;
  int mode = SG_FULL;       // products: SG_FULL / SG_SYM / SG_SYMSKEW
  int tiles = 0;            // items per block (filled in by the launcher)
  unsigned deps = 0;        // bit d: reads job d's output for the same block
  // products: C = epilogue(op(A) op(B) [+ alpha2 op(A2) op(B2)]), as SgemmArgs
  // expand: A = theta, C = Q;  pack: A = matrix, C = dtheta
  // symcomb: X = {A, B} (nin), outputs {C, C2, add_out[0], add_out[1]} (nout),
  //          Cb_f = transposed copy of A (optional)
  const float* A = nullptr;
  const float* B = nullptr;
  const float* A2 = nullptr;
  const float* B2 = nullptr;
  int a_sym = 0, a2_sym = 0;
  float alpha = 1.f, alpha2 = 1.f;
  float* C = nullptr;
  __nv_bfloat16* Cb = nullptr;
  float* C2 = nullptr;
  float alpha_c2 = 0.f, diag = 0.f, diag2 = 0.f;
  int nadd = 0;
  const float* add[4] = {nullptr, nullptr, nullptr, nullptr};
  float addc[4] = {0, 0, 0, 0};
  float addc2[4] = {0, 0, 0, 0};
  const float* skew_add = nullptr;
  float skew_c = 0.f;
  int nin = 0, nout = 0;
  float coef[4][2] = {{0, 0}, {0, 0}, {0, 0}, {0, 0}};
  float* add_out[2] = {nullptr, nullptr};
  float* Cb_f = nullptr;
};

struct CnpGraph {
  CnpJob job[kCnpMaxJobs];
  int njobs = 0, nblk = 0, b = 0;
  int item_start[kCnpMaxJobs + 1] = {0};
  int* counters = nullptr;  // scratch: njobs * nblk done-counters + 1 ticket
  int* err = nullptr;
  unsigned long long wait_ns = 0;  // bound of every dependency wait
  // initial value of the done-counter of job 0, block 0 (0 in every product call; the
  // wait-timeout self-test starts it far below reach so that the first dependent item's
  // wait runs out)
  int first_counter = 0;
};
// Zeroes the counters and runs the graph (two launches).
cudaError_t launch_cnp_graph(CnpGraph g, cudaStream_t s);

// ---- tcgen05 GEMM (kernels_umma.cu) ----------------------------------------------
// D[M x N] = A[M x K] . B[N x K]^T per batch entry, bf16 operands, fp32 accumulation.
// Operand X is K-major when X[row, k] is contiguous in k, MN-major when contiguous in
// the row index.  Each operand is a 2-D row-major bf16 matrix in global memory plus
// per-batch coordinate offsets.
struct UmmaOperand {
  const void* ptr = nullptr;  // base of the row-major 2-D matrix
  int64_t rows = 0, cols = 0; // extent of the 2-D matrix
  int64_t ld = 0;             // row stride in elements
  int mn_major = 0;           // 0: rows index M/N and cols index K; 1: rows index K
  int64_t boff_mn = 0;        // per-batch offset added to the M (or N) coordinate
  int64_t boff_k = 0;         // per-batch offset added to the K coordinate
};
struct UmmaGemm {
  UmmaOperand A, B;
  int M = 0, N = 0, K = 0, batch = 1;
  int ksplit = 1;             // split of K into ksplit partial sums (fp32 output only)
  void* D = nullptr;          // output base
  int out_f32 = 0;            // 0: bf16 output, 1: fp32 output
  int64_t ldd = 0;            // row stride of D in elements
  int64_t d_boff_col = 0;     // per-batch column offset of D
  int64_t d_boff = 0;         // per-batch element offset of D
  int64_t d_split = 0;        // per-split element offset of D
  int64_t d_cols = 0;         // columns of D (0: ldd); D may start inside a wider matrix
  // optional side job of two extra warps per CTA, run alongside the GEMM:
  // side_dst[r][c] = bf16(side_scales[r] * side_q[r][c]) for r < side_rows, c < side_cols
  // (the int8 weight's next panel while this panel is multiplied); side_rows = 0: none
  const int8_t* side_q = nullptr;
  int64_t side_ldq = 0;
  const float* side_scales = nullptr;
  void* side_dst = nullptr;
  int64_t side_ldd = 0;
  int side_rows = 0, side_cols = 0;
};
cudaError_t launch_umma_gemm(const UmmaGemm& g, const char* family, cudaStream_t s);
// The CTA-pair form (kernels_umma2.cu) for the plain merged-weight GEMMs: one batch entry,
// no K split, A K-major, bf16 output, N % 256 == 0, dense output (ldd == N).
bool umma_pair_eligible(const UmmaGemm& g);
cudaError_t launch_umma_gemm_pair(const UmmaGemm& g, const char* family, cudaStream_t s);
// whether launch_umma_gemm sends eligible GEMMs to the CTA-pair kernel (default: yes)
bool gemm_pairs_enabled();

// The CTA-pair GEMM with B from the int8 weight q (per-row scales; row stride ldq): B is the
// bf16 merged weight that g.B describes, each tile converted to bf16(s * q) in shared memory
// between its int8 load and the MMAs (no scratch).
struct PairQ8 {
  const int8_t* q = nullptr;  // W0q, row stride ldq (a multiple of 16)
  int64_t ldq = 0;
  const float* scales = nullptr;
};
cudaError_t launch_umma_gemm_pair_q8(const UmmaGemm& g, const PairQ8& q, const char* family,
                                     cudaStream_t s);
// ksplit the launcher would choose for the given problem (used to size scratch).
int umma_choose_ksplit(int M, int N, int K, int batch);

}  // namespace poetx
