/*
 * poetx.h -- C ABI of libpoetx, the B200 (sm_100a) implementation of the POET-X
 * orthogonal-equivalence linear layer.
 *
 * The layer (POET abstract: every weight is W = R W0 P with R, P learnable orthogonal
 * and W0 fixed and random; POET-X technical summary, section 2):
 *
 *     y = (Pi_R^T G_R Pi_R) W0 (Pi_P^T G_P Pi_P) x
 *
 *   - G_P, G_R are block-diagonal with b x b blocks built by the Cayley-Neumann
 *     parameterisation (section 2.4) from packed upper-triangular parameters theta;
 *   - Pi_P, Pi_R are fixed random permutations applied through index maps, never as
 *     matrices (section 2.2, permutation acceleration);
 *   - the inner two permutations are merged once into W0' = Pi_R W0 Pi_P^T (section
 *     2.2, permutation reduction), so a token row is processed input-centrically
 *     (section 2.1) as
 *         U = X[:, p_P];  V_j = U_j G_P,j^T;  W = V W0'^T;  Z_j = W_j G_R,j^T;
 *         Y[:, p_R[i]] = Z[:, i]
 *     and R W0 P is never formed.
 *
 * Conventions (the pages leave them open; these are the readings this library uses)
 *   permutation   int32 vector p; (Pi x)_i = x[p[i]]; inverse inv[p[i]] = i.
 *   blocks        block j covers coordinates [j*b, (j+1)*b) of the permuted space;
 *                 n % b == 0 and m % b == 0.
 *   theta         [nblk, b(b-1)/2] fp32, strict upper triangle row-major per block:
 *                 idx(i,j) = i*b - i*(i+1)/2 + (j-i-1) for i < j; Q_ij = theta,
 *                 Q_ji = -theta, Q_ii = 0.
 *   CNP           G = (I + Q)(I + Q + ... + Q^k) = I + 2(Q + ... + Q^k) + Q^(k+1).
 *   layouts       row-major: X [T, n], Y [T, m], W0 and W0' [m, n] (out x in),
 *                 G [nblk, b, b], dG [nblk, b, b].
 *   W0            frozen: the backward returns dX and dG (and, through
 *                 poetx_cnp_bwd, dtheta) but no dW0.
 *
 * Precision
 *   POETX_F32   everything fp32 (SIMT FFMA kernels).
 *   POETX_BF16  activations, W0, W0' and G operands bf16 (tcgen05 tensor cores, fp32
 *               accumulation in TMEM); theta, CNP, dG and dtheta fp32.  V, W, Z, dW,
 *               dV, dU intermediates are stored in bf16.  Supported b: 128, 256, 512.
 *
 * Memory and streams
 *   All pointers marked "device" are caller-owned device memory; the library never
 *   allocates.  Scratch comes from (ws, ws_bytes); the *_workspace() queries return
 *   the bytes a call needs.  Every device pointer must be 16-byte aligned.  All work is
 *   enqueued asynchronously on `stream` (a cudaStream_t; NULL = legacy default stream).
 *
 * Errors
 *   Every call returns a poetx_status.  Arguments are validated before anything is
 *   launched; a failed validation launches nothing.  poetx_last_error() gives detail
 *   text for the calling thread.  Launch failures map to POETX_ERR_CUDA.  Kernels that
 *   wait on barriers give up after a time limit, record POETX_ERR_TIMEOUT in a device
 *   flag and return; poetx_device_status() reads (and clears) that flag.
 */
#ifndef POETX_H
#define POETX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum poetx_status {
  POETX_OK = 0,
  POETX_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad flag */
  POETX_ERR_SHAPE = 2,       /* n % b or m % b nonzero, unsupported b or k */
  POETX_ERR_DTYPE = 3,       /* dtype not POETX_F32 / POETX_BF16 */
  POETX_ERR_ALIGN = 4,       /* a device pointer is not 16-byte aligned */
  POETX_ERR_WORKSPACE = 5,   /* ws_bytes below what the call needs */
  POETX_ERR_CUDA = 6,        /* a CUDA runtime call or launch failed */
  POETX_ERR_TIMEOUT = 7      /* a kernel's bounded barrier wait ran out */
} poetx_status;

enum { POETX_F32 = 0, POETX_BF16 = 1 };

/* Short description of a status code (static string). */
const char* poetx_status_string(int status);

/* Detail text of the last failed call on this thread ("" if none). */
const char* poetx_last_error(void);

/* Library version string. */
const char* poetx_version(void);

/*
 * Seeded random permutation of {0..n-1} and its inverse, in HOST memory.
 * POET-X section 2.2: the orthogonal factors carry fixed random permutations that are
 * applied by index maps.  Generator: SplitMix64 (Steele, Lea & Flood 2014) from `seed`,
 * Durstenfeld Fisher-Yates for i = n-1..1 with j = floor(r * (i+1) / 2^64).
 *   perm, inv: caller-owned host arrays of n int32 (inv may be NULL).
 *   Errors: POETX_ERR_INVALID_ARG if n < 0 or perm is NULL with n > 0.
 */
int poetx_make_perm(uint64_t seed, int32_t n, int32_t* perm, int32_t* inv);

/*
 * Inverse of a given index map, in HOST memory (POET-X section 2.2: Pi^T is applied as the
 * gather by the inverse map, inv[perm[i]] = i).  The map is checked first: every entry must
 * lie in [0, n) and appear once (a bijection), else nothing is written.
 *   perm: caller-owned host array of n int32, read.  inv: host array of n int32, written;
 *   must not be perm.
 *   Errors: POETX_ERR_INVALID_ARG for n < 0, NULL arrays with n > 0, perm == inv, an entry
 *   out of range or repeated (the detail text names it).
 */
int poetx_invert_perm(const int32_t* perm, int32_t n, int32_t* inv);

/*
 * Permutation reduction (POET-X section 2.2): W0' = Pi_R W0 Pi_P^T, i.e.
 * W0p[i, j] = W0[perm_R[i], perm_P[j]].  Run once per outer iteration.
 *   W0   device [m, n] (dtype), read.      W0p  device [m, n] (dtype), written.
 *   perm_R device int32 [m], perm_P device int32 [n].
 *   Bit-exact copy.  Errors: INVALID_ARG, DTYPE, ALIGN, CUDA.
 */
int poetx_merge_perm(const void* W0, void* W0p, int32_t m, int32_t n, const int32_t* perm_R,
                     const int32_t* perm_P, int dtype, void* stream);

/*
 * Outer-loop merge and re-initialisation.  The original POET step W <- R_i W P_i (POET-X
 * technical summary section 2.1, the weight-centric update that the input-centric layer
 * replaces inside an inner loop) folds the rotations of a finished inner loop into the
 * frozen weight; the next inner loop starts from theta = 0 under fresh permutations:
 *   M = G_R W0' G_P                 two batched block-diagonal products (block i of G_R
 *                                   acts on rows [ib, (i+1)b), block j of G_P on columns)
 *   W0p_new[i, j] = M[inv_R[perm_R_new[i]], inv_P[perm_P_new[j]]]
 * i.e. W0p_new = Pi_R' (R W0 P) Pi_P'^T with R = Pi_R^T G_R Pi_R, P = Pi_P^T G_P Pi_P.
 * The caller sets theta to zero afterwards (G = I); this call does not touch theta.
 *   W0p        device [m, n] (dtype): merged weight of the current permutations, read.
 *   G_P, G_R   device [n/b, b, b], [m/b, b, b] (dtype: the bf16 copies for POETX_BF16,
 *              fp32 for POETX_F32), read.
 *   inv_P, inv_R           device int32 [n], [m]: inverses of the current permutations.
 *   perm_P_new, perm_R_new device int32 [n], [m]: the next permutations.
 *   W0p_new    device [m, n] (dtype), written; must not alias W0p.
 *   ws         device scratch of poetx_outer_merge_workspace(m, n, dtype) bytes.
 * bf16: tcgen05 products with fp32 accumulation; G_R W0' and M are rounded to bf16 (as
 * the layer's activations are).  fp32: SIMT fp32 products.
 * Shapes: m % b == 0, n % b == 0; bf16 also needs b % 128 == 0.  All pointers 16-byte
 * aligned.  Errors: INVALID_ARG, SHAPE, DTYPE, ALIGN, WORKSPACE, CUDA.
 */
size_t poetx_outer_merge_workspace(int32_t m, int32_t n, int dtype);
int poetx_outer_merge(const void* W0p, const void* G_P, const void* G_R, int32_t m, int32_t n,
                      int32_t b, const int32_t* inv_P, const int32_t* inv_R,
                      const int32_t* perm_P_new, const int32_t* perm_R_new, void* W0p_new,
                      int dtype, void* ws, size_t ws_bytes, void* stream);

/*
 * Index-map permutation of the columns of a row-major matrix (POET-X section 2.2,
 * permutation acceleration): out[t, i] = in[t, idx[i]] for t < rows, i < cols.
 * With idx = perm this applies Pi to every row; with idx = inv it applies Pi^T.
 *   in, out device [rows, cols] (dtype), distinct buffers.  idx device int32 [cols].
 *   Bit-exact.  Errors: INVALID_ARG, DTYPE, ALIGN, CUDA.
 */
int poetx_permute_cols(const void* in, void* out, const int32_t* idx, int32_t rows, int32_t cols,
                       int dtype, void* stream);

/*
 * Scratch bytes needed by poetx_cnp_fwd / poetx_cnp_bwd for nblk blocks of size b with
 * Neumann order k (the calls also accept less, down to one block's worth, and then work
 * through the blocks in more chunks).  Returns 0 for invalid arguments.
 */
size_t poetx_cnp_workspace(int32_t nblk, int32_t b, int32_t k);

/*
 * Cayley-Neumann forward (POET-X section 2.4): for every block,
 *   Q = skew(theta),  G = (I + Q)(I + Q + ... + Q^k).
 *   theta   device fp32 [nblk, b(b-1)/2], read.
 *   G       device fp32 [nblk, b, b], written.
 *   G_bf16  device bf16 [nblk, b, b], written when non-NULL (the MMA operand copy,
 *           round-to-nearest-even of G).
 *   1 <= b <= 1024, 1 <= k <= 16.   fp32 throughout (SIMT FFMA).
 *   Errors: INVALID_ARG, SHAPE, ALIGN, WORKSPACE, CUDA.
 */
int poetx_cnp_fwd(const float* theta, float* G, void* G_bf16, int32_t nblk, int32_t b, int32_t k,
                  void* ws, size_t ws_bytes, void* stream);

/*
 * Cayley-Neumann forward without a caller scratch buffer.  The papers have no
 * counterpart: this entry point exists for callers that cannot allocate device memory
 * where they need G (a host framework that owns all device memory in its own pool and
 * exposes none to this call site, or a loop that must not call cudaMalloc because it
 * would synchronise the device).  Same arguments and result as poetx_cnp_fwd (bit for
 * bit: the same kernels on the same chunks of blocks), minus (ws, ws_bytes).
 *   Scratch: a fixed 32 MiB array of the library's own device memory, present on every
 *   GPU that loads the library until the process exits.  One block's forward scratch must
 *   fit it: (d + 2) b x b fp32 matrices plus 64 bytes of counters and a fixed 256 bytes,
 *   with d = floor((k + 1) / 2) -- every k <= 16 for b <= 512, k <= 10 for b = 1024;
 *   b = 1024 with k >= 11 returns POETX_ERR_WORKSPACE with a message.  Any number of
 *   blocks is processed in chunks.
 *   Set-up: the first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call before any
 *   stream capture.  The call allocates nothing and calls no allocating routine.
 *   Sharing: every call on a device uses the same array, which keeps the last call's
 *   contents; nothing in it needs to start at zero (each intermediate is fully written
 *   before it is read).  Calls whose GPU work overlaps (e.g. on two streams) race on
 *   the array: order them on one stream or with events.
 *   Errors: INVALID_ARG, SHAPE, ALIGN, WORKSPACE, CUDA.
 */
int poetx_cnp_fwd_static(const float* theta, float* G, void* G_bf16, int32_t nblk, int32_t b,
                         int32_t k, void* stream);

/*
 * Cayley-Neumann backward (POET-X section 2.4, backward optimised the same way as the
 * forward): dtheta = d<dG, G(theta)>/dtheta for the truncated polynomial as computed,
 *   dtheta_idx(i,j) = dQ_ij - dQ_ji.
 *   theta   device fp32 [nblk, b(b-1)/2], read.   dG device fp32 [nblk, b, b], read.
 *   dtheta  device fp32 [nblk, b(b-1)/2], written (overwritten, not accumulated).
 *   Errors: INVALID_ARG, SHAPE, ALIGN, WORKSPACE, CUDA.
 */
int poetx_cnp_bwd(const float* theta, const float* dG, float* dtheta, int32_t nblk, int32_t b,
                  int32_t k, void* ws, size_t ws_bytes, void* stream);

/*
 * The same CNP pair with the forward's Q, S = Q^2 and F' kept for the backward (POET-X
 * technical summary section 2.5 trades recomputation against memory the same way for the
 * layer's activations): with theta unchanged between the two calls, the backward reads
 * Q, S and F' instead of expanding theta and recomputing Q^2, the higher powers and F',
 * and its result is bit-identical to poetx_cnp_bwd.  F' = F(S) - f_0 I, where
 * G = E(S) + Q F(S) splits the CNP polynomial into its even and odd parts in Q (f_0 = 2,
 * the coefficient of Q).
 *   Q_save, S_save, F_save     device fp32 [nblk, b, b] each, written by poetx_cnp_fwd_save.
 *   Q_saved, S_saved, F_saved  the same buffers, read by poetx_cnp_bwd_saved.
 *   Other arguments and errors as poetx_cnp_fwd / poetx_cnp_bwd (a NULL save buffer with
 *   nblk > 0: INVALID_ARG).
 */
int poetx_cnp_fwd_save(const float* theta, float* G, void* G_bf16, float* Q_save, float* S_save,
                       float* F_save, int32_t nblk, int32_t b, int32_t k, void* ws,
                       size_t ws_bytes, void* stream);
int poetx_cnp_bwd_saved(const float* theta, const float* dG, const float* Q_saved,
                        const float* S_saved, const float* F_saved, float* dtheta, int32_t nblk,
                        int32_t b, int32_t k, void* ws, size_t ws_bytes, void* stream);

/* Shape, precision and index maps of one POET-X linear (index maps in device memory). */
typedef struct poetx_linear_desc {
  int32_t T;              /* tokens (rows of X and Y), >= 0 */
  int32_t n;              /* input features */
  int32_t m;              /* output features */
  int32_t b;              /* block size of G_P and G_R */
  int32_t dtype;          /* POETX_F32 or POETX_BF16 */
  const int32_t* perm_P;  /* device int32 [n] */
  const int32_t* inv_P;   /* device int32 [n] */
  const int32_t* perm_R;  /* device int32 [m] */
  const int32_t* inv_R;   /* device int32 [m] */
} poetx_linear_desc;

/* Scratch bytes of poetx_linear_fwd / poetx_linear_bwd.  The flags say which of the
 * optional save buffers the call will get (a missing one is kept in scratch or
 * recomputed).  Returns 0 for an invalid descriptor. */
size_t poetx_linear_fwd_workspace(const poetx_linear_desc* d, int has_save_u, int has_save_w);
size_t poetx_linear_bwd_workspace(const poetx_linear_desc* d, int has_save_u, int has_save_w);

/*
 * POET-X linear forward, input-centric with two index-map permutations.
 *   x      device [T, n] (dtype), read.
 *   G_P    device [n/b, b, b] (dtype: fp32 for POETX_F32, bf16 for POETX_BF16), read.
 *   G_R    device [m/b, b, b] (same), read.
 *   W0p    device [m, n] (dtype), the merged weight from poetx_merge_perm, read.
 *   y      device [T, m] (dtype), written.
 *   save_u device [T, n] or NULL: receives U = X[:, p_P] for the backward.
 *   save_w device [T, m] or NULL: receives W = V W0'^T for the backward (POET-Xfast);
 *          NULL together with NULL in the backward gives the recompute mode (POET-Xmem).
 *   T = 0 is a no-op.  Errors: INVALID_ARG, SHAPE, DTYPE, ALIGN, WORKSPACE, CUDA.
 */
int poetx_linear_fwd(const poetx_linear_desc* d, const void* x, const void* G_P, const void* G_R,
                     const void* W0p, void* y, void* save_u, void* save_w, void* ws,
                     size_t ws_bytes, void* stream);

/*
 * POET-X linear backward for the loss gradient dy (W0' frozen):
 *   dZ = dY[:, p_R]; dW_j = dZ_j G_R,j; dG_R,j = dZ_j^T W_j; dV = dW W0';
 *   dU_j = dV_j G_P,j; dG_P,j = dV_j^T U_j; dX[:, p_P[i]] = dU[:, i].
 *   x, dy        device [T, n], [T, m] (dtype), read.
 *   G_P, G_R, W0p  as in the forward, read.
 *   save_u, save_w the forward's save buffers, or NULL to recompute U (a gather) and
 *                W (block product + W0' GEMM) inside the call.
 *   dx           device [T, n] (dtype), written.
 *   dG_P, dG_R   device fp32 [n/b, b, b], [m/b, b, b]; overwritten when accumulate = 0,
 *                added to when accumulate = 1 (micro-batch accumulation; dG is linear in
 *                the tokens).  The token sums are reduced in a fixed order (no float
 *                atomics), so results are identical from run to run.
 *   Errors: INVALID_ARG, SHAPE, DTYPE, ALIGN, WORKSPACE, CUDA.
 */
int poetx_linear_bwd(const poetx_linear_desc* d, const void* x, const void* dy, const void* G_P,
                     const void* G_R, const void* W0p, const void* save_u, const void* save_w,
                     void* dx, float* dG_P, float* dG_R, int accumulate, void* ws,
                     size_t ws_bytes, void* stream);

/*
 * Int8 base weight (POET-X technical summary section 2.6, POET-XQ: training on a low-bit
 * base model, whose weight is dequantised on the fly only where it is needed and never
 * stored in high precision).  The pages give no scheme; here one fp32 scale per output
 * channel (row of W0'):
 *   scales[i] = max_j |W[i, j]| / 127,   q[i, j] = round_to_nearest_even(W[i, j] / scales[i])
 * clamped to [-127, 127] (an all-zero row: scale 0, codes 0).  Scale and codes are decided
 * in fp32 with IEEE division, so they are reproducible bit for bit.
 *   W       device [m, n] (dtype POETX_BF16 or POETX_F32), read.
 *   q       device int8 [m, n], written.     scales  device fp32 [m], written.
 *   Errors: INVALID_ARG, DTYPE, ALIGN, CUDA.
 */
int poetx_quantize_rows(const void* W, int8_t* q, float* scales, int32_t m, int32_t n, int dtype,
                        void* stream);

/*
 * Permutation reduction straight into the int8 merged weight (POET-X section 2.2 with the
 * section 2.6 base weight): the codes and scales that poetx_quantize_rows gives for
 * W0' = Pi_R W0 Pi_P^T, bit for bit, without forming W0' in high precision.  A permutation
 * of a row does not change its largest magnitude, so row i's scale is that of source row
 * perm_R[i]; each source row is staged on chip and gathered there.
 *   W0 device [m, n] (dtype POETX_BF16 or POETX_F32), read; perm_R device int32 [m],
 *   perm_P device int32 [n]; W0q device int8 [m, n], scales device fp32 [m], written.
 *   Rows up to 200 KB (n * element size).  Errors: INVALID_ARG, SHAPE, DTYPE, ALIGN, CUDA.
 */
int poetx_merge_perm_q8(const void* W0, int8_t* W0q, float* scales, int32_t m, int32_t n,
                        const int32_t* perm_R, const int32_t* perm_P, int dtype, void* stream);

/*
 * The bf16 layer with the int8 merged weight (codes and scales from poetx_merge_perm_q8 or
 * poetx_quantize_rows of W0').  The weight is dequantised where the two W0' GEMMs use it,
 * bf16(scales[i] * q[i, j]) (fp32 product, round to nearest even): the tensor-core kernel
 * loads each weight tile as int8 and converts it in shared memory just before its MMAs, so
 * no bf16 copy of the weight is written to device memory.  Shapes the CTA-pair kernel does
 * not take (N % 256 != 0, fewer than 256 tokens, n % 16 != 0, or pairs switched off with
 * poetx_set_gemm_pairs) instead dequantise one panel of the weight at a time (at most 32 MB
 * of bf16, at most a quarter of the weight when its N allows) into scratch and multiply it.
 * The first poetx_linear_q8_scratch(d) bytes of ws hold that panel buffer; the rest is the
 * layer call's scratch, so ws_bytes must be at least poetx_linear_q8_scratch(d) +
 * poetx_linear_{fwd,bwd}_workspace(d, ...).  Results equal poetx_linear_fwd / _bwd run on
 * the dequantised weight.
 *   W0q device int8 [m, n], scales device fp32 [m]: read.  Other arguments as the bf16
 *   entry points.  d->dtype must be POETX_BF16 (else DTYPE).
 *   Errors: as poetx_linear_fwd / poetx_linear_bwd.
 */
size_t poetx_linear_q8_scratch(const poetx_linear_desc* d);
int poetx_linear_fwd_q8(const poetx_linear_desc* d, const void* x, const void* G_P,
                        const void* G_R, const int8_t* W0q, const float* scales, void* y,
                        void* save_u, void* save_w, void* ws, size_t ws_bytes, void* stream);
int poetx_linear_bwd_q8(const poetx_linear_desc* d, const void* x, const void* dy,
                        const void* G_P, const void* G_R, const int8_t* W0q, const float* scales,
                        const void* save_u, const void* save_w, void* dx, float* dG_P,
                        float* dG_R, int accumulate, void* ws, size_t ws_bytes, void* stream);

/*
 * Time limit of every bounded wait in the library's kernels (mbarrier waits of the tensor-core
 * GEMM, dependency waits of the CNP task graph), in nanoseconds; 0 restores the default of
 * 2 s.  Kernels read the limit when they are launched (a CUDA graph keeps the value it was
 * captured with).  Not thread-safe against concurrent launches that expect the old value.
 *   previous: receives the limit before this call (may be NULL).
 *   Errors: POETX_ERR_INVALID_ARG above 60 s.
 */
int poetx_set_wait_limit(uint64_t ns, uint64_t* previous);

/*
 * Kernel choice for the merged-weight GEMMs (W = V W0'^T, dV = dW W0'): 1 (the default)
 * runs them on CTA pairs (tcgen05 cta_group::2, 256 x 256 tiles shared by two SMs) when
 * the shape allows (N % 256 == 0, M >= 256); 0 runs them on single CTAs (128 x 256 tiles).
 * The block-diagonal and dG products always run on single CTAs.  Both forms compute the
 * same products; the switch exists to compare them.  Applies to launches made after the
 * call.
 *   previous: receives the setting before this call (may be NULL).
 *   Errors: POETX_ERR_INVALID_ARG for a value other than 0 or 1.
 */
int poetx_set_gemm_pairs(int enable, int* previous);

/*
 * Self-test of the bounded waits (no counterpart in the pages): runs the CNP forward task
 * graph of nblk blocks with the done-counter of block 0's first step started far below
 * reach, so the first item that depends on it waits until the time limit, records
 * POETX_ERR_TIMEOUT in the device flag and the launch returns.  Nothing faults and nothing
 * waits without a bound; G holds partial results afterwards.  poetx_device_status then
 * reports (and clears) the timeout, and later calls run normally.
 *   theta device fp32 [nblk, b(b-1)/2], G device fp32 [nblk, b, b] (written, partially).
 *   ws: scratch holding every block at once: nblk * (d + 2) b x b fp32 matrices (d =
 *   floor((k + 1) / 2)) plus 64 bytes of counters per block and 256 bytes;
 *   poetx_cnp_workspace(nblk, b, k) is enough whenever nblk * b * b * 4 <= 256 MiB.
 *   Shapes: b % 64 == 0 and k <= 6 (the task-graph shapes), nblk >= 1.
 *   Errors: INVALID_ARG, SHAPE, ALIGN, WORKSPACE, CUDA.
 */
int poetx_selftest_wait_timeout(const float* theta, float* G, int32_t nblk, int32_t b, int32_t k,
                                void* ws, size_t ws_bytes, void* stream);

/*
 * FP32 FMA throughput probe (no counterpart in the pages; the measured peak of the pipe that
 * bounds the SIMT CNP kernels): one launch of `ctas` CTAs x 512 threads, every thread running
 * 16 independent chains of `iters` fused multiply-adds (in packed pairs, two FMAs per
 * instruction), i.e. ctas * 512 * 16 * iters * 2 FLOPs.  Time it with events on `stream`.
 *   out: device fp32 [ctas * 512], written (the chains' sums).
 *   Errors: INVALID_ARG, ALIGN, CUDA.
 */
int poetx_fma_probe(float* out, int32_t ctas, int32_t iters, void* stream);

/*
 * Reads and clears the device-side error flag that kernels with bounded barrier waits
 * set on a timeout.  Synchronises the given stream first.  Returns POETX_OK or
 * POETX_ERR_TIMEOUT (or POETX_ERR_CUDA if the synchronisation itself failed).
 */
int poetx_device_status(void* stream);

/*
 * Launch accounting and per-kernel timing.
 *   poetx_launch_count() counts every kernel launch the library has made.
 *   poetx_profile_begin(name) starts bracketing every launch of the kernel family
 *   `name` ("gemm_w0", "gemm_blockdiag", "gemm_dG", "permute", "cnp_sgemm", ...) with
 *   CUDA events on the launch stream (NULL or "" turns this off); poetx_profile_end()
 *   stops bracketing, synchronises those events and reports the number of bracketed
 *   launches and their summed device time in milliseconds.  Launches made while the
 *   stream is captured into a CUDA graph get event nodes in the graph: each replay of the
 *   graph records them again, and a further poetx_profile_end() (without a new
 *   poetx_profile_begin) reports the launches of the latest replay.  Events come from a
 *   fixed pool of 32768 pairs; launches beyond it are not bracketed (the count reports
 *   how many were).
 */
uint64_t poetx_launch_count(void);
int poetx_profile_begin(const char* name);
int poetx_profile_end(int32_t* launches, double* total_ms);

#ifdef __cplusplus
}
#endif

#endif /* POETX_H */
