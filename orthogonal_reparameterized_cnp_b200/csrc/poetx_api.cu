// C ABI of libpoetx: argument validation, the permutation generator, scratch layout and
// the launch sequences of the POET-X layer (POET-X technical summary, section 2).
#include <cuda_runtime.h>

#include <atomic>
#include <initializer_list>
#include <utility>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "poetx_internal.h"

namespace poetx {

// ------------------------------------------------------------------ errors
static thread_local std::string g_last_error;

void set_error(const std::string& msg) { g_last_error = msg; }
int fail(int status, const std::string& msg) {
  g_last_error = msg;
  return status;
}
int cuda_fail(cudaError_t e, const char* what) {
  g_last_error = std::string(what) + ": " + cudaGetErrorString(e);
  return POETX_ERR_CUDA;
}

// Device-side error flag: kernels with bounded waits record POETX_ERR_TIMEOUT here.
__device__ int g_device_error = 0;

int* device_error_flag() {
  static int* ptrs[64] = {nullptr};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return nullptr;
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<int*>(p);
  }
  return ptrs[dev];
}

static std::atomic<unsigned long long> g_wait_limit_ns{2000000000ull};  // 2 s

unsigned long long wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

static std::atomic<int> g_gemm_pairs{1};
bool gemm_pairs_enabled() { return g_gemm_pairs.load(std::memory_order_relaxed) != 0; }

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!cache[dev]) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = v > 0 ? v : 148;
  }
  return cache[dev];
}

// ------------------------------------------------------------------ launch accounting
static std::atomic<uint64_t> g_launches{0};
static std::mutex g_prof_mu;
static std::string g_prof_family;
static bool g_prof_on = false;
static constexpr int kEventPairs = 32768;
static std::vector<cudaEvent_t> g_ev_start, g_ev_stop;
static int g_prof_used = 0;

// While a stream is being captured into a CUDA graph the events are recorded as event
// nodes of the graph (cudaEventRecordExternal), so every replay of the graph re-records
// them and the elapsed times describe the launches of the latest replay.
static void record_event(cudaEvent_t ev, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal);
  else
    cudaEventRecord(ev, s);
}

void begin_launch(const char* family, cudaStream_t s) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (!g_prof_on) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (g_prof_on && g_prof_family == family && g_prof_used < kEventPairs)
    record_event(g_ev_start[g_prof_used], s);
}
void end_launch(const char* family, cudaStream_t s) {
  if (!g_prof_on) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (g_prof_on && g_prof_family == family && g_prof_used < kEventPairs)
    record_event(g_ev_stop[g_prof_used++], s);
}

// ------------------------------------------------------------------ helpers
namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

size_t align_up(size_t v, size_t a = 256) { return (v + a - 1) / a * a; }

struct Carve {
  char* base;
  size_t off = 0;
  explicit Carve(void* b) : base(static_cast<char*>(b)) {}
  void* take(size_t bytes) {
    void* p = base ? base + off : nullptr;
    off += align_up(bytes);
    return p;
  }
};

#define POETX_CUDA(call, what)                 \
  do {                                         \
    cudaError_t e_ = (call);                   \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)

// ---- CNP polynomial coefficients ---------------------------------------------------
// G = sum_{i=0..k+1} c_i Q^i with c = (1, 2, ..., 2, 1).  With S = Q^2 (symmetric):
//   G = E(S) + Q F(S),  E = sum_j e_j S^j (e_j = c_{2j}),  F = sum_j f_j S^j (f_j = c_{2j+1})
// E is symmetric and Q F skew, so G's upper triangle gives both halves.
struct CnpPoly {
  int d;          // highest power of S needed: floor((k+1)/2)
  float e[10], f[10];
};
CnpPoly cnp_poly(int k) {
  CnpPoly p;
  p.d = (k + 1) / 2;
  for (int j = 0; j <= p.d; ++j) {
    auto c = [&](int i) -> float {
      if (i < 0 || i > k + 1) return 0.f;
      return (i == 0 || i == k + 1) ? 1.f : 2.f;
    };
    p.e[j] = c(2 * j);
    p.f[j] = c(2 * j + 1);
  }
  return p;
}

// Matrices held per block in the CNP scratch (b x b fp32 each).
int cnp_mats(int k, bool backward) {
  const int d = (k + 1) / 2;
  // forward: Q, P_1..P_d, F'
  // backward adds: D, dG^T, N_1..N_d, Pm, R, R2, T, T2, A
  return backward ? 2 * d + 10 : d + 2;
}

constexpr size_t kCnpChunkTarget = 256ull << 20;  // bytes per scratch matrix

// per block: the matrices plus the task graph's done-counters (<= 16 jobs)
constexpr size_t kCnpCounterBytesPerBlock = 64;
constexpr size_t kCnpFixedBytes = 256;

size_t cnp_per_block(int b, int k, bool backward) {
  return (size_t)cnp_mats(k, backward) * align_up((size_t)b * b * 4) + kCnpCounterBytesPerBlock;
}

// The one-launch task graph covers square blocks with b % 64 == 0 and k <= 6.
bool cnp_graph_ok(int b, int k) { return b >= 64 && b % 64 == 0 && (k + 1) / 2 <= 3; }

int cnp_validate(const void* theta, const void* out, int nblk, int b, int k) {
  if (nblk < 0) return fail(POETX_ERR_INVALID_ARG, "nblk must be >= 0");
  if (b < 1 || b > 1024) return fail(POETX_ERR_SHAPE, "block size b must be in [1, 1024]");
  if (k < 1 || k > 16) return fail(POETX_ERR_SHAPE, "Neumann order k must be in [1, 16]");
  if (nblk > 0 && (!theta || !out)) return fail(POETX_ERR_INVALID_ARG, "null pointer");
  return POETX_OK;
}

// The scratch rules every CNP call checks (one block's worth at least, non-null, aligned),
// also where a path needs none, so that the contract does not depend on the path.
int cnp_ws_check(int b, int k, bool backward, const void* ws, size_t ws_bytes) {
  const size_t per = cnp_per_block(b, k, backward);
  const size_t cap = ws_bytes > kCnpFixedBytes ? (ws_bytes - kCnpFixedBytes) / per : 0;
  if (cap < 1) return fail(POETX_ERR_WORKSPACE, "CNP scratch smaller than one block needs");
  if (!ws) return fail(POETX_ERR_INVALID_ARG, "null scratch");
  if (!aligned16(ws)) return fail(POETX_ERR_ALIGN, "scratch must be 16-byte aligned");
  return POETX_OK;
}

// Runs fn(first_block, count, scratch) over chunks of blocks that fit in ws.
template <typename Fn>
int cnp_chunks(int nblk, int b, int k, bool backward, void* ws, size_t ws_bytes, Fn fn) {
  const int st = cnp_ws_check(b, k, backward, ws, ws_bytes);
  if (st != POETX_OK) return st;
  const size_t per = cnp_per_block(b, k, backward);
  size_t cap = (ws_bytes - kCnpFixedBytes) / per;
  const size_t per_mat_cap = kCnpChunkTarget / ((size_t)b * b * 4);
  if (cap > per_mat_cap && per_mat_cap >= 1) cap = per_mat_cap;
  for (int b0 = 0; b0 < nblk; b0 += (int)cap) {
    int cnt = nblk - b0 < (int)cap ? nblk - b0 : (int)cap;
    int st = fn(b0, cnt);
    if (st != POETX_OK) return st;
  }
  return POETX_OK;
}

}  // namespace

size_t cnp_fwd_block_bytes(int b, int k) { return cnp_per_block(b, k, false); }
size_t cnp_fixed_bytes() { return kCnpFixedBytes; }

namespace {

SgemmArgs sq_gemm(const float* A, int tA, const float* B, int tB, float* C, int nb, int b,
                  int mode) {
  SgemmArgs g;
  const int64_t bb = (int64_t)b * b;
  g.A = A; g.lda = b; g.sA = bb; g.transA = tA;
  g.B = B; g.ldb = b; g.sB = bb; g.transB = tB;
  g.C = C; g.ldc = b; g.sC = bb;
  g.M = b; g.N = b; g.K = b; g.batch = nb;
  g.mode = mode;
  return g;
}

}  // namespace
}  // namespace poetx

using namespace poetx;

// ======================================================================= C ABI
extern "C" {

const char* poetx_status_string(int status) {
  switch (status) {
    case POETX_OK: return "ok";
    case POETX_ERR_INVALID_ARG: return "invalid argument";
    case POETX_ERR_SHAPE: return "unsupported or inconsistent shape";
    case POETX_ERR_DTYPE: return "unsupported dtype";
    case POETX_ERR_ALIGN: return "pointer not 16-byte aligned";
    case POETX_ERR_WORKSPACE: return "workspace too small";
    case POETX_ERR_CUDA: return "CUDA error";
    case POETX_ERR_TIMEOUT: return "device wait timed out";
    default: return "unknown status";
  }
}

const char* poetx_last_error(void) { return g_last_error.c_str(); }

const char* poetx_version(void) { return "poetx 0.1.0 (sm_100a)"; }

int poetx_make_perm(uint64_t seed, int32_t n, int32_t* perm, int32_t* inv) {
  if (n < 0) return fail(POETX_ERR_INVALID_ARG, "n must be >= 0");
  if (n > 0 && !perm) return fail(POETX_ERR_INVALID_ARG, "perm is NULL");
  for (int32_t i = 0; i < n; ++i) perm[i] = i;
  // SplitMix64 stream feeding Durstenfeld's Fisher-Yates; bounded draw by the high word
  // of a 64x64 -> 128-bit product (Lemire's multiply-shift, no rejection).
  uint64_t state = seed;
  for (int32_t i = n - 1; i >= 1; --i) {
    state += 0x9E3779B97F4A7C15ull;
    uint64_t z = state;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    z ^= z >> 31;
    const uint64_t j = (uint64_t)(((unsigned __int128)z * (unsigned __int128)(uint64_t)(i + 1)) >> 64);
    int32_t t = perm[i];
    perm[i] = perm[j];
    perm[j] = t;
  }
  if (inv)
    for (int32_t i = 0; i < n; ++i) inv[perm[i]] = i;
  return POETX_OK;
}

int poetx_invert_perm(const int32_t* perm, int32_t n, int32_t* inv) {
  if (n < 0) return fail(POETX_ERR_INVALID_ARG, "n must be >= 0");
  if (n == 0) return POETX_OK;
  if (!perm || !inv) return fail(POETX_ERR_INVALID_ARG, "perm and inv must be given");
  if (perm == inv) return fail(POETX_ERR_INVALID_ARG, "perm and inv must be distinct arrays");
  // every index in range and taken once: the map is a bijection of {0..n-1}
  std::vector<unsigned char> seen((size_t)n, 0);
  for (int32_t i = 0; i < n; ++i) {
    const int32_t p = perm[i];
    if (p < 0 || p >= n)
      return fail(POETX_ERR_INVALID_ARG, "perm[" + std::to_string(i) + "] = " +
                                             std::to_string(p) + " is outside [0, n)");
    if (seen[(size_t)p])
      return fail(POETX_ERR_INVALID_ARG, "perm is not a bijection: index " + std::to_string(p) +
                                             " appears twice");
    seen[(size_t)p] = 1;
  }
  for (int32_t i = 0; i < n; ++i) inv[perm[i]] = i;
  return POETX_OK;
}

int poetx_set_gemm_pairs(int enable, int* previous) {
  if (enable != 0 && enable != 1) return fail(POETX_ERR_INVALID_ARG, "enable must be 0 or 1");
  const int old = g_gemm_pairs.exchange(enable);
  if (previous) *previous = old;
  return POETX_OK;
}

int poetx_set_wait_limit(uint64_t ns, uint64_t* previous) {
  if (ns > 60ull * 1000000000ull)
    return fail(POETX_ERR_INVALID_ARG, "wait limit above 60 s");
  const unsigned long long v = ns ? ns : 2000000000ull;
  const unsigned long long old = g_wait_limit_ns.exchange(v);
  if (previous) *previous = old;
  return POETX_OK;
}

int poetx_merge_perm(const void* W0, void* W0p, int32_t m, int32_t n, const int32_t* perm_R,
                     const int32_t* perm_P, int dtype, void* stream) {
  if (m < 0 || n < 0) return fail(POETX_ERR_INVALID_ARG, "negative size");
  if (dtype != POETX_F32 && dtype != POETX_BF16) return fail(POETX_ERR_DTYPE, "bad dtype");
  if (m == 0 || n == 0) return POETX_OK;
  if (!W0 || !W0p || !perm_R || !perm_P) return fail(POETX_ERR_INVALID_ARG, "null pointer");
  if (W0 == W0p) return fail(POETX_ERR_INVALID_ARG, "W0 and W0p must be distinct");
  if (!aligned16(W0) || !aligned16(W0p) || !aligned16(perm_R) || !aligned16(perm_P))
    return fail(POETX_ERR_ALIGN, "pointers must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  POETX_CUDA(launch_gather(W0, W0p, perm_R, perm_P, m, n, n, n, dtype == POETX_BF16 ? 2 : 4, s),
             "merge_perm launch");
  return POETX_OK;
}

int poetx_permute_cols(const void* in, void* out, const int32_t* idx, int32_t rows, int32_t cols,
                       int dtype, void* stream) {
  if (rows < 0 || cols < 0) return fail(POETX_ERR_INVALID_ARG, "negative size");
  if (dtype != POETX_F32 && dtype != POETX_BF16) return fail(POETX_ERR_DTYPE, "bad dtype");
  if (rows == 0 || cols == 0) return POETX_OK;
  if (!in || !out || !idx) return fail(POETX_ERR_INVALID_ARG, "null pointer");
  if (in == out) return fail(POETX_ERR_INVALID_ARG, "in and out must be distinct");
  if (!aligned16(in) || !aligned16(out) || !aligned16(idx))
    return fail(POETX_ERR_ALIGN, "pointers must be 16-byte aligned");
  POETX_CUDA(launch_gather(in, out, nullptr, idx, rows, cols, cols, cols,
                           dtype == POETX_BF16 ? 2 : 4, static_cast<cudaStream_t>(stream)),
             "permute launch");
  return POETX_OK;
}

size_t poetx_cnp_workspace(int32_t nblk, int32_t b, int32_t k) {
  if (nblk < 0 || b < 1 || b > 1024 || k < 1 || k > 16) return 0;
  if (nblk == 0) return 0;
  const size_t per_mat_cap = kCnpChunkTarget / ((size_t)b * b * 4);
  size_t chunk = (size_t)nblk;
  if (per_mat_cap >= 1 && chunk > per_mat_cap) chunk = per_mat_cap;
  return chunk * cnp_per_block(b, k, true) + kCnpFixedBytes;
}

}  // extern "C"

namespace {

// P_1 = Q Q, P_p = S P_{p-1} (all symmetric), and F' = F - f_0 I = sum_{j>=1} f_j P_j
// produced as the second output of the last power product.
int cnp_powers(const float* Q, std::vector<float*>& Pw, float* Fp, const CnpPoly& P, int nb,
               int b, cudaStream_t s) {
  const int d = P.d;
  for (int j = 1; j <= d; ++j) {
    SgemmArgs g = (j == 1) ? sq_gemm(Q, 0, Q, 0, Pw[1], nb, b, SG_SYM)
                           : sq_gemm(Pw[1], 0, Pw[j - 1], 0, Pw[j], nb, b, SG_SYM);
    g.a_sym = (j == 1) ? -1 : 1;  // Q is skew, S symmetric
    if (j == d) {
      g.C2 = Fp;
      g.alpha_c2 = P.f[d];
      for (int t = 1; t < d; ++t) {
        g.add[g.nadd] = Pw[t];
        g.addc[g.nadd] = 0.f;
        g.addc2[g.nadd] = P.f[t];
        ++g.nadd;
      }
    }
    POETX_CUDA(launch_sgemm(g, s), "cnp power product");
  }
  return POETX_OK;
}

// ---- the task-graph form of the CNP (one persistent launch per chunk) -------------
CnpJob prod_job(const float* A, int a_sym, const float* B, float* C, int mode, unsigned deps) {
  CnpJob j;
  j.type = JOB_PRODUCT;
  j.mode = mode;
  j.A = A;
  j.a_sym = a_sym;
  j.B = B;
  j.C = C;
  j.deps = deps;
  return j;
}

// powers P_1 = Q Q, P_p = S P_{p-1}.  The last product emits, instead of P_d itself,
//   C  = E(S) = e_0 I + sum_{j>=1} e_j P_j     and     C2 = F' = sum_{j>=1} f_j P_j,
// so later steps read one tile for each polynomial (for d = 1 the single product keeps
// C = S, which the backward reads, and E is formed where it is used).
// Returns the job index of P_j in idx[j].
void graph_powers(CnpGraph& g, int jQ, const float* Q, float* const* Pw, float* Fp,
                  const CnpPoly& P, int* idx, int j_first = 1, int j_last = -1) {
  const int d = P.d;
  if (j_last < 0) j_last = d;
  for (int j = j_first; j <= j_last; ++j) {
    CnpJob jb = (j == 1) ? prod_job(Q, -1, Q, Pw[1], SG_SYM, 1u << jQ)
                         : prod_job(Pw[1], 1, Pw[j - 1], Pw[j], SG_SYM,
                                    (1u << idx[1]) | (1u << idx[j - 1]));
    if (j == d) {
      jb.C2 = Fp;
      jb.alpha_c2 = P.f[d];
      if (d >= 2) {
        jb.alpha = P.e[d];
        jb.diag = P.e[0];
      }
      for (int t = 1; t < d; ++t) {
        jb.add[jb.nadd] = Pw[t];
        jb.addc[jb.nadd] = P.e[t];
        jb.addc2[jb.nadd] = P.f[t];
        ++jb.nadd;
        jb.deps |= 1u << idx[t];
      }
    }
    idx[j] = g.njobs;
    g.job[g.njobs++] = jb;
  }
}

int run_fwd_graph(const float* theta, const float* Q, float* const* Pw, float* Fp, float* G,
                  __nv_bfloat16* Gb, int* counters, const CnpPoly& P, int nb, int b,
                  cudaStream_t s, int first_counter = 0) {
  const int d = P.d;
  CnpGraph g;
  g.nblk = nb;
  g.b = b;
  g.counters = counters;
  g.first_counter = first_counter;
  CnpJob ex;
  ex.type = JOB_EXPAND;
  ex.A = theta;
  ex.C = const_cast<float*>(Q);
  g.job[g.njobs++] = ex;
  int idx[4] = {0, 0, 0, 0};
  graph_powers(g, 0, Q, Pw, Fp, P, idx);
  // G = E + f_0 Q + Q F' (upper tiles; E symmetric, QF skew); E is the last power job's
  // output for d >= 2, else e_0 I + e_1 S
  CnpJob jg = prod_job(Q, -1, Fp, G, SG_SYMSKEW, 1u | (1u << idx[d]));
  jg.Cb = Gb;
  jg.add[0] = Pw[d];
  jg.addc[0] = d >= 2 ? 1.f : P.e[1];
  jg.diag = d >= 2 ? 0.f : P.e[0];
  jg.nadd = 1;
  jg.skew_add = Q;
  jg.skew_c = P.f[0];
  g.job[g.njobs++] = jg;
  POETX_CUDA(launch_cnp_graph(g, s), "cnp graph (forward)");
  return POETX_OK;
}

struct BwdMats {
  float *Q, *P[4], *Fp, *D, *dGt, *N[4], *Pm, *R, *R2, *T, *T2, *A;
  bool saved = false;  // Q, P[1] = S and Fp = F' are given (from the forward)
};

int run_bwd_graph(const float* theta, const float* dg, float* dtheta, const BwdMats& M,
                  int* counters, const CnpPoly& P, int nb, int b, cudaStream_t s) {
  const int d = P.d;
  CnpGraph g;
  g.nblk = nb;
  g.b = b;
  g.counters = counters;
  // with Q, S and F' saved by the forward there is no expansion and there are no power
  // jobs; otherwise job 0 expands theta into Q
  if (!M.saved) {
    CnpJob ex;
    ex.type = JOB_EXPAND;
    ex.A = theta;
    ex.C = M.Q;
    g.job[g.njobs++] = ex;
  }
  const unsigned dQ = M.saved ? 0u : 1u;  // dependency bit on Q
  int idx[4] = {0, 0, 0, 0};
  // jobs are queued level by level so independent work is not stuck behind tiles that
  // wait: S and D (both need only Q), then the higher powers, then the Horner terms.
  if (!M.saved) graph_powers(g, 0, M.Q, M.P, M.Fp, P, idx, 1, 1);
  // D = Q dG (the adjoint reaching F is Q^T dG = -D)
  const int jD = g.njobs;
  g.job[g.njobs++] = prod_job(M.Q, -1, dg, M.D, SG_FULL, dQ);
  if (!M.saved && d >= 2) graph_powers(g, 0, M.Q, M.P, M.Fp, P, idx, 2, d);
  // dependency bits on S and on F' (none when they are inputs)
  const unsigned dS = M.saved ? 0u : 1u << idx[1];
  const unsigned dF = M.saved ? 0u : 1u << idx[d];
  // N_j = e_j (dG + dG^T) - f_j (D + D^T), j = 1..d, and dG^T
  const int jN = g.njobs;
  {
    CnpJob jn;
    jn.type = JOB_SYMCOMB;
    jn.A = dg;
    jn.B = M.D;
    jn.nin = 2;
    jn.nout = d;
    jn.C = M.N[1];
    jn.C2 = d >= 2 ? M.N[2] : nullptr;
    jn.add_out[0] = d >= 3 ? M.N[3] : nullptr;
    for (int o = 0; o < d; ++o) {
      jn.coef[o][0] = P.e[o + 1];
      jn.coef[o][1] = -P.f[o + 1];
    }
    jn.Cb_f = M.dGt;
    jn.deps = 1u << jD;
    g.job[g.njobs++] = jn;
  }
  // Y = sum_j sum_a S^a N_j S^(j-1-a)
  const float* Y = M.N[1];
  int jY = jN;
  const float* S = M.P[1];
  if (d >= 2) {
    // T_{d-2} = N_{d-1} + S N_d + N_d S: symmetric (S N_d is the transpose of N_d S), so one
    // structured job of two products over the upper tiles, mirrored
    const int jT = g.njobs;
    CnpJob jt = prod_job(S, 1, M.N[d], M.T, SG_SYM, (1u << jN) | dS);
    jt.A2 = M.N[d];
    jt.a2_sym = 1;
    jt.B2 = S;
    jt.alpha2 = 1.f;
    jt.add[0] = M.N[d - 1];
    jt.addc[0] = 1.f;
    jt.nadd = 1;
    g.job[g.njobs++] = jt;
    Y = M.T;
    jY = jT;
    if (d == 3) {
      // transposed Horner terms keep every A operand symmetric:
      //   Rt_1 = N_2 + S N_3,  Rt_0 = N_1 + S Rt_1,  T_0 = Rt_0 + T_1 S
      const int jR1 = g.njobs;
      CnpJob r1 = prod_job(S, 1, M.N[3], M.R, SG_FULL, dS | (1u << jN));
      r1.add[0] = M.N[2];
      r1.addc[0] = 1.f;
      r1.nadd = 1;
      g.job[g.njobs++] = r1;
      const int jR0 = g.njobs;
      CnpJob r0 = prod_job(S, 1, M.R, M.R2, SG_FULL, dS | (1u << jN) | (1u << jR1));
      r0.add[0] = M.N[1];
      r0.addc[0] = 1.f;
      r0.nadd = 1;
      g.job[g.njobs++] = r0;
      const int jT0 = g.njobs;
      CnpJob t0 = prod_job(M.T, 1, S, M.T2, SG_SYM, (1u << jT) | dS | (1u << jR0));
      t0.add[0] = M.R2;
      t0.addc[0] = 1.f;
      t0.nadd = 1;
      g.job[g.njobs++] = t0;
      Y = M.T2;
      jY = jT0;
    }
  }
  // A = f_0 dG + dG F' - Y Q; dtheta_(i,j) = A_ij - A_ji
  const int jA = g.njobs;
  CnpJob ja = prod_job(M.dGt, 2, M.Fp, M.A, SG_FULL, dQ | (1u << jN) | dF | (1u << jY));
  ja.A2 = Y;
  ja.a2_sym = 1;
  ja.B2 = M.Q;
  ja.alpha2 = -1.f;
  ja.add[0] = dg;
  ja.addc[0] = P.f[0];
  ja.nadd = 1;
  g.job[g.njobs++] = ja;
  CnpJob pk;
  pk.type = JOB_PACK;
  pk.A = M.A;
  pk.C = dtheta;
  pk.deps = 1u << jA;
  g.job[g.njobs++] = pk;
  POETX_CUDA(launch_cnp_graph(g, s), "cnp graph (backward)");
  return POETX_OK;
}

}  // namespace

extern "C" {

// Q_save / S_save / F_save (optional, all or none): receive Q, S = Q^2 and F' per block.
static int cnp_fwd_impl(const float* theta, float* G, void* G_bf16, float* Q_save, float* S_save,
                        float* F_save, int32_t nblk, int32_t b, int32_t k, void* ws,
                        size_t ws_bytes, void* stream) {
  int st = cnp_validate(theta, G, nblk, b, k);
  if (st != POETX_OK) return st;
  if (nblk == 0) return POETX_OK;
  if (!aligned16(theta) || !aligned16(G) || (G_bf16 && !aligned16(G_bf16)) ||
      !aligned16(Q_save) || !aligned16(S_save) || !aligned16(F_save))
    return fail(POETX_ERR_ALIGN, "pointers must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cnp_fused_ok(b, k)) {  // every block on chip: one launch, the scratch is not used
    const int wst = cnp_ws_check(b, k, false, ws, ws_bytes);
    if (wst != POETX_OK) return wst;
    POETX_CUDA(launch_cnp_fused_fwd(theta, G, G_bf16, Q_save, S_save, F_save, nblk, b, k, s),
               "cnp fused forward");
    return POETX_OK;
  }
  const CnpPoly P = cnp_poly(k);
  const int d = P.d;
  const int64_t bb = (int64_t)b * b, ntri = (int64_t)b * (b - 1) / 2;
  return cnp_chunks(nblk, b, k, false, ws, ws_bytes, [&](int b0, int nb) -> int {
    Carve cv(ws);
    float* Q = static_cast<float*>(cv.take(bb * 4 * nb));
    std::vector<float*> Pw(d + 1, nullptr);
    for (int j = 1; j <= d; ++j) Pw[j] = static_cast<float*>(cv.take(bb * 4 * nb));
    float* Fp = static_cast<float*>(cv.take(bb * 4 * nb));
    if (S_save) {  // the saved matrices are written in place of the scratch copies
      Q = Q_save + b0 * bb;
      Pw[1] = S_save + b0 * bb;
      Fp = F_save + b0 * bb;
    }
    if (cnp_graph_ok(b, k)) {
      int* counters = static_cast<int*>(cv.take(kCnpCounterBytesPerBlock * nb + 4));
      __nv_bfloat16* Gb =
          G_bf16 ? static_cast<__nv_bfloat16*>(G_bf16) + b0 * bb : nullptr;
      return run_fwd_graph(theta + b0 * ntri, Q, Pw.data(), Fp, G + b0 * bb, Gb, counters, P,
                           nb, b, s);
    }
    POETX_CUDA(launch_theta_to_Q(theta + b0 * ntri, Q, nb, b, s), "cnp theta->Q");
    int st2 = cnp_powers(Q, Pw, Fp, P, nb, b, s);
    if (st2 != POETX_OK) return st2;
    // G = E + Q F with E = e_0 I + sum_j e_j P_j (symmetric) and Q F = Q F' + f_0 Q (skew):
    // only upper tiles are multiplied; G_ji = E_ij - (QF)_ij.
    SgemmArgs g = sq_gemm(Q, 0, Fp, 0, G + b0 * bb, nb, b, SG_SYMSKEW);
    g.a_sym = -1;
    g.C_bf16 = G_bf16 ? static_cast<void*>(static_cast<uint16_t*>(G_bf16) + b0 * bb) : nullptr;
    g.diag = P.e[0];
    for (int j = 1; j <= d; ++j) {
      g.add[g.nadd] = Pw[j];
      g.addc[g.nadd] = P.e[j];
      ++g.nadd;
    }
    g.skew_add = Q;
    g.skew_c = P.f[0];
    POETX_CUDA(launch_sgemm(g, s), "cnp G");
    return POETX_OK;
  });
}

int poetx_cnp_fwd(const float* theta, float* G, void* G_bf16, int32_t nblk, int32_t b, int32_t k,
                  void* ws, size_t ws_bytes, void* stream) {
  return cnp_fwd_impl(theta, G, G_bf16, nullptr, nullptr, nullptr, nblk, b, k, ws, ws_bytes,
                      stream);
}

int poetx_cnp_fwd_save(const float* theta, float* G, void* G_bf16, float* Q_save, float* S_save,
                       float* F_save, int32_t nblk, int32_t b, int32_t k, void* ws,
                       size_t ws_bytes, void* stream) {
  if (nblk > 0 && (!Q_save || !S_save || !F_save))
    return fail(POETX_ERR_INVALID_ARG, "null pointer");
  return cnp_fwd_impl(theta, G, G_bf16, Q_save, S_save, F_save, nblk, b, k, ws, ws_bytes,
                      stream);
}

// Q_saved / S_saved / F_saved (optional, all or none): Q, S and F' of the forward on the
// same theta.
static int cnp_bwd_impl(const float* theta, const float* dG, const float* Q_saved,
                        const float* S_saved, const float* F_saved, float* dtheta, int32_t nblk,
                        int32_t b, int32_t k, void* ws, size_t ws_bytes, void* stream) {
  int st = cnp_validate(theta, dtheta, nblk, b, k);
  if (st != POETX_OK) return st;
  if (nblk == 0) return POETX_OK;
  if (!dG) return fail(POETX_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(theta) || !aligned16(dG) || !aligned16(dtheta) || !aligned16(Q_saved) ||
      !aligned16(S_saved) || !aligned16(F_saved))
    return fail(POETX_ERR_ALIGN, "pointers must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cnp_fused_ok(b, k)) {
    const int wst = cnp_ws_check(b, k, true, ws, ws_bytes);
    if (wst != POETX_OK) return wst;
    POETX_CUDA(launch_cnp_fused_bwd(theta, dG, Q_saved, S_saved, F_saved, dtheta, nblk, b, k, s),
               "cnp fused backward");
    return POETX_OK;
  }
  const CnpPoly P = cnp_poly(k);
  const int d = P.d;
  const int64_t bb = (int64_t)b * b, ntri = (int64_t)b * (b - 1) / 2;
  return cnp_chunks(nblk, b, k, true, ws, ws_bytes, [&](int b0, int nb) -> int {
    Carve cv(ws);
    auto mat = [&]() { return static_cast<float*>(cv.take(bb * 4 * nb)); };
    float* Q = mat();
    std::vector<float*> Pw(d + 1, nullptr), Nw(d + 1, nullptr);
    for (int j = 1; j <= d; ++j) Pw[j] = mat();
    float* Fp = mat();
    float* D = mat();
    float* dGt = mat();
    for (int j = 1; j <= d; ++j) Nw[j] = mat();
    float* Pm = mat();
    float* R = mat();
    float* R2 = mat();
    float* T = mat();
    float* T2 = mat();
    float* A = mat();
    const float* dg = dG + b0 * bb;
    const bool saved = S_saved != nullptr;
    if (saved) {  // Q, S and F' come from the forward (read only)
      Q = const_cast<float*>(Q_saved) + b0 * bb;
      Pw[1] = const_cast<float*>(S_saved) + b0 * bb;
      Fp = const_cast<float*>(F_saved) + b0 * bb;
    }
    if (cnp_graph_ok(b, k)) {
      int* counters = static_cast<int*>(cv.take(kCnpCounterBytesPerBlock * nb + 4));
      BwdMats M;
      M.Q = Q;
      for (int j = 0; j < 4; ++j) {
        M.P[j] = j <= d ? Pw[j] : nullptr;
        M.N[j] = j <= d ? Nw[j] : nullptr;
      }
      M.Fp = Fp; M.D = D; M.dGt = dGt; M.Pm = Pm; M.R = R; M.R2 = R2; M.T = T; M.T2 = T2;
      M.A = A;
      M.saved = saved;
      return run_bwd_graph(theta + b0 * ntri, dg, dtheta + b0 * ntri, M, counters, P, nb, b, s);
    }
    if (!saved) {
      POETX_CUDA(launch_theta_to_Q(theta + b0 * ntri, Q, nb, b, s), "cnp theta->Q");
      int st2 = cnp_powers(Q, Pw, Fp, P, nb, b, s);
      if (st2 != POETX_OK) return st2;
    }
    // D = Q dG; the adjoint reaching F is Q^T dG = -D.
    {
      SgemmArgs gd = sq_gemm(Q, 0, dg, 0, D, nb, b, SG_FULL);
      gd.a_sym = -1;
      POETX_CUDA(launch_sgemm(gd, s), "cnp D");
    }
    // N_j = M_j + M_j^T with M_j = e_j dG - f_j D  (upstream of S^j through E and F)
    for (int j0 = 1; j0 <= d; j0 += 4) {
      const int cnt = (d - j0 + 1) < 4 ? (d - j0 + 1) : 4;
      const float* X[2] = {dg, D};
      float* outs[4];
      float coef[8];
      for (int t = 0; t < cnt; ++t) {
        outs[t] = Nw[j0 + t];
        coef[t * 2 + 0] = P.e[j0 + t];
        coef[t * 2 + 1] = -P.f[j0 + t];
      }
      POETX_CUDA(launch_symcomb(X, 2, outs, cnt, coef, nb, b, s, j0 == 1 ? dGt : nullptr),
                 "cnp N");
    }
    // Y = dS + dS^T = sum_j sum_a S^a N_j S^(j-1-a), by a Horner recursion from the top
    const float* Y = Nw[1];
    if (d >= 2) {
      const float* S = Pw[1];
      SgemmArgs g = sq_gemm(Nw[d], 0, S, 0, Pm, nb, b, SG_FULL);  // Pm = N_d S
      g.a_sym = 1;
      if (d >= 3) {  // R_{d-2} = N_{d-1} + Pm
        g.C2 = R;
        g.alpha_c2 = 1.f;
        g.add[0] = Nw[d - 1];
        g.addc[0] = 0.f;
        g.addc2[0] = 1.f;
        g.nadd = 1;
      }
      POETX_CUDA(launch_sgemm(g, s), "cnp N_d S");
      {  // T_{d-2} = N_{d-1} + Pm + Pm^T
        const float* X[2] = {Nw[d - 1], Pm};
        float* outs[1] = {T};
        float coef[2] = {0.5f, 1.f};
        POETX_CUDA(launch_symcomb(X, 2, outs, 1, coef, nb, b, s), "cnp T");
      }
      float* Rc = R;
      float* Rn = R2;
      float* Tc = T;
      float* Tn = T2;
      for (int a = d - 3; a >= 0; --a) {
        // R_a = N_{a+1} + R_{a+1} S
        SgemmArgs gr = sq_gemm(Rc, 0, S, 0, Rn, nb, b, SG_FULL);
        gr.add[0] = Nw[a + 1];
        gr.addc[0] = 1.f;
        gr.nadd = 1;
        POETX_CUDA(launch_sgemm(gr, s), "cnp R");
        // T_a = R_a + S T_{a+1}  (symmetric: upper tiles + mirror)
        SgemmArgs gt = sq_gemm(S, 0, Tc, 0, Tn, nb, b, SG_SYM);
        gt.a_sym = 1;
        gt.add[0] = Rn;
        gt.addc[0] = 1.f;
        gt.nadd = 1;
        POETX_CUDA(launch_sgemm(gt, s), "cnp T");
        std::swap(Rc, Rn);
        std::swap(Tc, Tn);
      }
      Y = Tc;
    }
    // A = f_0 dG + dG F' - Y Q  (skew part of A gives dtheta)
    SgemmArgs ga = sq_gemm(dGt, 0, Fp, 0, A, nb, b, SG_FULL);
    ga.a_sym = 2;  // dGt holds dG^T, so dG is read by rows
    ga.A2 = Y; ga.lda2 = b; ga.sA2 = bb;
    ga.B2 = Q; ga.ldb2 = b; ga.sB2 = bb;
    ga.K2 = b;
    ga.alpha2 = -1.f;
    ga.a2_sym = 1;  // Y is symmetric
    ga.add[0] = dg;
    ga.addc[0] = P.f[0];
    ga.nadd = 1;
    POETX_CUDA(launch_sgemm(ga, s), "cnp A");
    POETX_CUDA(launch_pack_skew(A, dtheta + b0 * ntri, nb, b, s), "cnp pack");
    return POETX_OK;
  });
}

int poetx_cnp_bwd(const float* theta, const float* dG, float* dtheta, int32_t nblk, int32_t b,
                  int32_t k, void* ws, size_t ws_bytes, void* stream) {
  return cnp_bwd_impl(theta, dG, nullptr, nullptr, nullptr, dtheta, nblk, b, k, ws, ws_bytes,
                      stream);
}

int poetx_cnp_bwd_saved(const float* theta, const float* dG, const float* Q_saved,
                        const float* S_saved, const float* F_saved, float* dtheta, int32_t nblk,
                        int32_t b, int32_t k, void* ws, size_t ws_bytes, void* stream) {
  if (nblk > 0 && (!Q_saved || !S_saved || !F_saved))
    return fail(POETX_ERR_INVALID_ARG, "null pointer");
  return cnp_bwd_impl(theta, dG, Q_saved, S_saved, F_saved, dtheta, nblk, b, k, ws, ws_bytes,
                      stream);
}

int poetx_selftest_wait_timeout(const float* theta, float* G, int32_t nblk, int32_t b, int32_t k,
                                void* ws, size_t ws_bytes, void* stream) {
  int st = cnp_validate(theta, G, nblk, b, k);
  if (st != POETX_OK) return st;
  if (nblk < 1) return fail(POETX_ERR_INVALID_ARG, "nblk must be >= 1");
  if (!cnp_graph_ok(b, k))
    return fail(POETX_ERR_SHAPE, "the self-test needs the task-graph shapes (b % 64 == 0, k <= 6)");
  if (!aligned16(theta) || !aligned16(G)) return fail(POETX_ERR_ALIGN, "pointers must be 16-byte aligned");
  const size_t per = cnp_per_block(b, k, false);
  if (!ws || ws_bytes < (size_t)nblk * per + kCnpFixedBytes)
    return fail(POETX_ERR_WORKSPACE, "self-test scratch must hold every block (no chunking)");
  if (!aligned16(ws)) return fail(POETX_ERR_ALIGN, "scratch must be 16-byte aligned");
  const CnpPoly P = cnp_poly(k);
  const int d = P.d;
  const int64_t bb = (int64_t)b * b;
  Carve cv(ws);
  float* Q = static_cast<float*>(cv.take(bb * 4 * nblk));
  std::vector<float*> Pw(d + 1, nullptr);
  for (int j = 1; j <= d; ++j) Pw[j] = static_cast<float*>(cv.take(bb * 4 * nblk));
  float* Fp = static_cast<float*>(cv.take(bb * 4 * nblk));
  int* counters = static_cast<int*>(cv.take(kCnpCounterBytesPerBlock * nblk + 4));
  // the expansion of block 0 can never be counted as done, so the first item that reads
  // it waits until the time limit
  return run_fwd_graph(theta, Q, Pw.data(), Fp, G, nullptr, counters, P, nblk, b,
                       static_cast<cudaStream_t>(stream), INT32_MIN / 2);
}

}  // extern "C"

// ======================================================================= linear layer
namespace {

int linear_validate(const poetx_linear_desc* d) {
  if (!d) return fail(POETX_ERR_INVALID_ARG, "descriptor is NULL");
  if (d->T < 0 || d->n < 1 || d->m < 1 || d->b < 1)
    return fail(POETX_ERR_INVALID_ARG, "sizes must be T >= 0 and n, m, b >= 1");
  if (d->dtype != POETX_F32 && d->dtype != POETX_BF16) return fail(POETX_ERR_DTYPE, "bad dtype");
  if (d->n % d->b || d->m % d->b) return fail(POETX_ERR_SHAPE, "n and m must be multiples of b");
  if (d->dtype == POETX_BF16 && d->b != 128 && d->b != 256 && d->b != 512)
    return fail(POETX_ERR_SHAPE, "bf16 layer supports b in {128, 256, 512}");
  if (d->dtype == POETX_F32 && d->b > 1024) return fail(POETX_ERR_SHAPE, "b must be <= 1024");
  if (!d->perm_P || !d->inv_P || !d->perm_R || !d->inv_R)
    return fail(POETX_ERR_INVALID_ARG, "index maps must be given");
  if (!aligned16(d->perm_P) || !aligned16(d->inv_P) || !aligned16(d->perm_R) ||
      !aligned16(d->inv_R))
    return fail(POETX_ERR_ALIGN, "index maps must be 16-byte aligned");
  return POETX_OK;
}

int check_ptrs(std::initializer_list<const void*> ps) {
  for (const void* p : ps) {
    if (!p) return fail(POETX_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(p)) return fail(POETX_ERR_ALIGN, "pointers must be 16-byte aligned");
  }
  return POETX_OK;
}

int check_opt(const void* p) {
  if (p && !aligned16(p)) return fail(POETX_ERR_ALIGN, "pointers must be 16-byte aligned");
  return POETX_OK;
}

struct FwdLayout {
  size_t U, V, W, Z, total;
};
FwdLayout fwd_layout(const poetx_linear_desc* d, int has_u, int has_w) {
  const size_t es = d->dtype == POETX_BF16 ? 2 : 4;
  const size_t tn = (size_t)d->T * d->n * es, tm = (size_t)d->T * d->m * es;
  FwdLayout L;
  L.U = has_u ? 0 : align_up(tn);
  L.V = align_up(tn);
  L.W = has_w ? 0 : align_up(tm);
  L.Z = align_up(tm);
  L.total = L.U + L.V + L.W + L.Z;
  return L;
}

struct BwdLayout {
  size_t U, Vr, Wr, dZ, dW, dV, dU, partR, partP, total;
  int ksR, ksP;
};
BwdLayout bwd_layout(const poetx_linear_desc* d, int has_u, int has_w) {
  const size_t es = d->dtype == POETX_BF16 ? 2 : 4;
  const size_t tn = (size_t)d->T * d->n * es, tm = (size_t)d->T * d->m * es;
  const int nP = d->n / d->b, nR = d->m / d->b;
  BwdLayout L;
  L.U = has_u ? 0 : align_up(tn);
  L.Vr = has_w ? 0 : align_up(tn);
  L.Wr = has_w ? 0 : align_up(tm);
  L.dZ = align_up(tm);
  L.dW = align_up(tm);
  L.dV = align_up(tn);
  L.dU = align_up(tn);
  L.ksR = L.ksP = 1;
  L.partR = L.partP = 0;
  if (d->dtype == POETX_BF16 && d->T > 0) {
    L.ksR = umma_choose_ksplit(d->b, d->b, d->T, nR);
    L.ksP = umma_choose_ksplit(d->b, d->b, d->T, nP);
    L.partR = align_up((size_t)L.ksR * nR * d->b * d->b * 4);
    L.partP = align_up((size_t)L.ksP * nP * d->b * d->b * 4);
  }
  L.total = L.U + L.Vr + L.Wr + L.dZ + L.dW + L.dV + L.dU + L.partR + L.partP;
  return L;
}

// ---- fp32 building blocks (SIMT) --------------------------------------------------
// out[:, j*b:(j+1)*b] = in[:, j*b:(j+1)*b] . (G_j^T if transposeG else G_j)
cudaError_t f32_blockdiag(const float* in, const float* G, float* out, int T, int width, int b,
                          bool transposeG, cudaStream_t s) {
  SgemmArgs g;
  g.A = in; g.lda = width; g.sA = b; g.transA = 0;
  g.B = G; g.ldb = b; g.sB = (int64_t)b * b; g.transB = transposeG ? 1 : 0;
  g.C = out; g.ldc = width; g.sC = b;
  g.M = T; g.N = b; g.K = b; g.batch = width / b;
  return launch_sgemm(g, s);
}
// dG_j (+)= A_j^T B_j over the token axis, A, B [T, width] row-major
cudaError_t f32_block_grad(const float* A, const float* B, float* dG, int T, int width, int b,
                           int accumulate, cudaStream_t s) {
  SgemmArgs g;
  g.A = A; g.lda = width; g.sA = b; g.transA = 1;
  g.B = B; g.ldb = width; g.sB = b; g.transB = 0;
  g.C = dG; g.ldc = b; g.sC = (int64_t)b * b;
  g.M = b; g.N = b; g.K = T; g.batch = width / b;
  if (accumulate) {
    g.add[0] = dG;
    g.addc[0] = 1.f;
    g.nadd = 1;
  }
  return launch_sgemm(g, s);
}

// ---- bf16 building blocks (tcgen05) -----------------------------------------------
UmmaOperand act_kmajor(const void* p, int T, int width, int64_t boff_k) {
  UmmaOperand o;
  o.ptr = p; o.rows = T; o.cols = width; o.ld = width; o.mn_major = 0; o.boff_k = boff_k;
  return o;
}
UmmaOperand act_mnmajor(const void* p, int T, int width, int64_t boff_mn) {
  UmmaOperand o;
  o.ptr = p; o.rows = T; o.cols = width; o.ld = width; o.mn_major = 1; o.boff_mn = boff_mn;
  return o;
}
cudaError_t bf16_blockdiag(const void* in, const void* G, void* out, int T, int width, int b,
                           bool transposeG, cudaStream_t s) {
  const int nblk = width / b;
  UmmaGemm g;
  g.A = act_kmajor(in, T, width, b);
  UmmaOperand B;
  B.ptr = G; B.rows = (int64_t)nblk * b; B.cols = b; B.ld = b;
  if (!transposeG) {  // B[n=r][k=c] = G_j[r][c]: K-major
    B.mn_major = 0; B.boff_mn = b;
  } else {            // B[n=r][k=c] = G_j[c][r]: MN-major
    B.mn_major = 1; B.boff_k = b;
  }
  g.B = B;
  g.M = T; g.N = b; g.K = b; g.batch = nblk;
  g.D = out; g.out_f32 = 0; g.ldd = width; g.d_boff_col = b;
  // forward products use G^T (B K-major); backward products use G (B MN-major)
  return launch_umma_gemm(g, "gemm_blockdiag", s);
}
cudaError_t bf16_block_grad(const void* A, const void* B, float* part, float* dG, int ks, int T,
                            int width, int b, int accumulate, cudaStream_t s) {
  const int nblk = width / b;
  UmmaGemm g;
  g.A = act_mnmajor(A, T, width, b);
  g.B = act_mnmajor(B, T, width, b);
  g.M = b; g.N = b; g.K = T; g.batch = nblk; g.ksplit = ks;
  g.D = part; g.out_f32 = 1; g.ldd = b; g.d_boff = (int64_t)b * b;
  g.d_split = (int64_t)nblk * b * b;
  cudaError_t e = launch_umma_gemm(g, "gemm_dG", s);
  if (e != cudaSuccess) return e;
  return launch_split_reduce(part, ks, (int64_t)nblk * b * b, dG, (int64_t)nblk * b * b,
                             accumulate, s);
}
cudaError_t bf16_w0(const void* in, const void* W0p, void* out, int T, int n, int m, bool forward,
                    cudaStream_t s) {
  UmmaGemm g;
  if (forward) {  // W[T, m] = V[T, n] W0'^T : B[n=o][k=i] = W0'[o][i], K-major
    g.A = act_kmajor(in, T, n, 0);
    UmmaOperand B;
    B.ptr = W0p; B.rows = m; B.cols = n; B.ld = n; B.mn_major = 0;
    g.B = B;
    g.M = T; g.N = m; g.K = n;
    g.D = out; g.ldd = m;
  } else {        // dV[T, n] = dW[T, m] W0' : B[n=i][k=o] = W0'[o][i], MN-major
    g.A = act_kmajor(in, T, m, 0);
    UmmaOperand B;
    B.ptr = W0p; B.rows = m; B.cols = n; B.ld = n; B.mn_major = 1;
    g.B = B;
    g.M = T; g.N = n; g.K = m;
    g.D = out; g.ldd = n;
  }
  g.batch = 1;
  g.out_f32 = 0;
  return launch_umma_gemm(g, "gemm_w0", s);
}

// The merged weight of a layer call: bf16 W0' (q == nullptr), or its int8 codes with per-row
// scales (the int8 layer) plus one bf16 panel buffer for the shapes that the CTA-pair kernel
// does not take.
struct W0Ref {
  const void* bf16 = nullptr;
  const int8_t* q = nullptr;
  const float* s = nullptr;
  void* panel = nullptr;
  int panel_f = 0, panel_b = 0;  // panel widths (along N) of the forward / backward GEMMs
};

// Panels of the int8 weight along the GEMM's N: a multiple of 256, at most 32 MB of bf16
// (K x width x 2 bytes), and at most a quarter of N (so two panels never hold more than half
// of the weight) where N allows.
constexpr size_t kPanelBytes = 32ull << 20;
int q8_panel_width(int N, int K) {
  int64_t w = (int64_t)(kPanelBytes / ((size_t)K * 2)) / 256 * 256;
  const int64_t quarter = (int64_t)N / 4 / 256 * 256;
  if (quarter >= 256 && w > quarter) w = quarter;
  if (w < 256) w = 256;
  const int64_t nr = ((int64_t)N + 255) / 256 * 256;
  return (int)(w < nr ? w : nr);
}
struct Q8Layout {
  int panel_f, panel_b;
  size_t panel_bytes, total;
};
Q8Layout q8_layout(const poetx_linear_desc* d) {
  Q8Layout L;
  L.panel_f = q8_panel_width(d->m, d->n);  // forward: N = m rows of W0', K = n
  L.panel_b = q8_panel_width(d->n, d->m);  // backward: N = n columns of W0', K = m
  const size_t ef = (size_t)L.panel_f * d->n, eb = (size_t)d->m * L.panel_b;
  L.panel_bytes = align_up((ef > eb ? ef : eb) * 2);
  L.total = L.panel_bytes;
  return L;
}

// W = V W0'^T (forward) or dV = dW W0' (backward) for either form of the weight.
cudaError_t w0_gemm(const void* in, const W0Ref& w, void* out, int T, int n, int m, bool forward,
                    cudaStream_t s) {
  if (!w.q) return bf16_w0(in, w.bf16, out, T, n, m, forward, s);
  // the GEMM as it reads the bf16 merged weight (B's pointer is not used)
  UmmaGemm g;
  UmmaOperand B;
  B.rows = m; B.cols = n; B.ld = n; B.mn_major = forward ? 0 : 1;
  g.A = act_kmajor(in, T, forward ? n : m, 0);
  g.B = B;
  g.M = T; g.N = forward ? m : n; g.K = forward ? n : m;
  g.batch = 1; g.out_f32 = 0;
  g.D = out; g.ldd = g.N;
  if (gemm_pairs_enabled() && umma_pair_eligible(g) && n % 16 == 0) {  // converted on chip
    PairQ8 q;
    q.q = w.q; q.ldq = n; q.scales = w.s;
    return launch_umma_gemm_pair_q8(g, q, "gemm_w0", s);
  }
  const int pw = forward ? w.panel_f : w.panel_b;
  // other shapes: panel by panel, each dequantised and then multiplied (one panel buffer)
  for (int p0 = 0; p0 < g.N; p0 += pw) {
    const int width = g.N - p0 < pw ? g.N - p0 : pw;
    cudaError_t e;
    UmmaGemm h = g;
    UmmaOperand P;
    if (forward) {  // rows p0.. of W0': [width x n]
      e = launch_dequant_2d(w.q + (int64_t)p0 * n, n, w.s + p0, w.panel, n, width, n, s);
      P.ptr = w.panel; P.rows = width; P.cols = n; P.ld = n; P.mn_major = 0;
    } else {        // columns p0.. of W0': [m x width]
      e = launch_dequant_2d(w.q + p0, n, w.s, w.panel, width, m, width, s);
      P.ptr = w.panel; P.rows = m; P.cols = width; P.ld = width; P.mn_major = 1;
    }
    if (e != cudaSuccess) return e;
    h.B = P;
    h.N = width;
    h.D = static_cast<__nv_bfloat16*>(out) + p0;
    h.ldd = g.N;
    h.d_cols = width;
    e = launch_umma_gemm(h, "gemm_w0", s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// Forward body shared by poetx_linear_fwd and the recompute path of the backward.
// Writes U (if U != x-gather target), V, W; Z and y only when y != nullptr.
int forward_body(const poetx_linear_desc* d, const void* x, const void* G_P, const void* G_R,
                 const W0Ref& w0, void* y, void* U, void* V, void* W, void* Z, cudaStream_t s) {
  const void* W0p = w0.bf16;
  const int T = d->T, n = d->n, m = d->m, b = d->b;
  const bool bf = d->dtype == POETX_BF16;
  const int es = bf ? 2 : 4;
  POETX_CUDA(launch_gather(x, U, nullptr, d->perm_P, T, n, n, n, es, s), "gather x");
  if (bf) {
    POETX_CUDA(bf16_blockdiag(U, G_P, V, T, n, b, false, s), "blockdiag G_P");
    POETX_CUDA(w0_gemm(V, w0, W, T, n, m, true, s), "W0' gemm");
    if (y) {
      POETX_CUDA(bf16_blockdiag(W, G_R, Z, T, m, b, false, s), "blockdiag G_R");
      POETX_CUDA(launch_gather(Z, y, nullptr, d->inv_R, T, m, m, m, es, s), "scatter y");
    }
  } else {
    POETX_CUDA(f32_blockdiag((const float*)U, (const float*)G_P, (float*)V, T, n, b, true, s),
               "blockdiag G_P");
    SgemmArgs g;
    g.A = (const float*)V; g.lda = n;
    g.B = (const float*)W0p; g.ldb = n; g.transB = 1;
    g.C = (float*)W; g.ldc = m;
    g.M = T; g.N = m; g.K = n; g.batch = 1;
    POETX_CUDA(launch_sgemm(g, s), "W0' gemm");
    if (y) {
      POETX_CUDA(f32_blockdiag((const float*)W, (const float*)G_R, (float*)Z, T, m, b, true, s),
                 "blockdiag G_R");
      POETX_CUDA(launch_gather(Z, y, nullptr, d->inv_R, T, m, m, m, es, s), "scatter y");
    }
  }
  return POETX_OK;
}

}  // namespace

extern "C" {

size_t poetx_linear_fwd_workspace(const poetx_linear_desc* d, int has_save_u, int has_save_w) {
  if (!d || d->T < 0 || d->n < 1 || d->m < 1 || d->b < 1) return 0;
  return fwd_layout(d, has_save_u, has_save_w).total;
}

size_t poetx_linear_bwd_workspace(const poetx_linear_desc* d, int has_save_u, int has_save_w) {
  if (!d || d->T < 0 || d->n < 1 || d->m < 1 || d->b < 1) return 0;
  return bwd_layout(d, has_save_u, has_save_w).total;
}

}  // extern "C"

namespace {
int linear_fwd_impl(const poetx_linear_desc* d, const void* x, const void* G_P, const void* G_R,
                    const W0Ref& w0, void* y, void* save_u, void* save_w, void* ws,
                    size_t ws_bytes, void* stream) {
  int st = linear_validate(d);
  if (st != POETX_OK) return st;
  if (d->T == 0) return POETX_OK;
  if ((st = check_ptrs({x, G_P, G_R, w0.q ? (const void*)w0.q : w0.bf16, y})) != POETX_OK)
    return st;
  if ((st = check_opt(save_u)) != POETX_OK || (st = check_opt(save_w)) != POETX_OK) return st;
  const FwdLayout L = fwd_layout(d, save_u != nullptr, save_w != nullptr);
  if (ws_bytes < L.total) return fail(POETX_ERR_WORKSPACE, "forward scratch too small");
  if (L.total && !ws) return fail(POETX_ERR_INVALID_ARG, "scratch is NULL");
  if ((st = check_opt(ws)) != POETX_OK) return st;
  Carve cv(ws);
  void* U = save_u ? save_u : cv.take(L.U);
  void* V = cv.take(L.V);
  void* W = save_w ? save_w : cv.take(L.W);
  void* Z = cv.take(L.Z);
  return forward_body(d, x, G_P, G_R, w0, y, U, V, W, Z, static_cast<cudaStream_t>(stream));
}

int linear_bwd_impl(const poetx_linear_desc* d, const void* x, const void* dy, const void* G_P,
                    const void* G_R, const W0Ref& w0, const void* save_u, const void* save_w,
                    void* dx, float* dG_P, float* dG_R, int accumulate, void* ws,
                    size_t ws_bytes, void* stream) {
  const void* W0p = w0.bf16;
  int st = linear_validate(d);
  if (st != POETX_OK) return st;
  if (accumulate != 0 && accumulate != 1)
    return fail(POETX_ERR_INVALID_ARG, "accumulate must be 0 or 1");
  if ((st = check_ptrs({dG_P, dG_R})) != POETX_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int T = d->T, n = d->n, m = d->m, b = d->b;
  const int nP = n / b, nR = m / b;
  if (T == 0) {  // empty token set: dG = 0 (or unchanged when accumulating)
    if (!accumulate) {
      POETX_CUDA(launch_split_reduce(nullptr, 0, 0, dG_P, (int64_t)nP * b * b, 0, s), "zero dG");
      POETX_CUDA(launch_split_reduce(nullptr, 0, 0, dG_R, (int64_t)nR * b * b, 0, s), "zero dG");
    }
    return POETX_OK;
  }
  if ((st = check_ptrs({dy, G_P, G_R, w0.q ? (const void*)w0.q : W0p, dx})) != POETX_OK)
    return st;
  if ((st = check_opt(save_u)) != POETX_OK || (st = check_opt(save_w)) != POETX_OK) return st;
  if (!save_u || !save_w)
    if ((st = check_ptrs({x})) != POETX_OK) return st;
  const BwdLayout L = bwd_layout(d, save_u != nullptr, save_w != nullptr);
  if (ws_bytes < L.total) return fail(POETX_ERR_WORKSPACE, "backward scratch too small");
  if (L.total && !ws) return fail(POETX_ERR_INVALID_ARG, "scratch is NULL");
  if ((st = check_opt(ws)) != POETX_OK) return st;
  const bool bf = d->dtype == POETX_BF16;
  const int es = bf ? 2 : 4;
  Carve cv(ws);
  void* U = save_u ? const_cast<void*>(save_u) : cv.take(L.U);
  void* Vr = save_w ? nullptr : cv.take(L.Vr);
  void* W = save_w ? const_cast<void*>(save_w) : cv.take(L.Wr);
  void* dZ = cv.take(L.dZ);
  void* dW = cv.take(L.dW);
  void* dV = cv.take(L.dV);
  void* dU = cv.take(L.dU);
  float* partR = static_cast<float*>(cv.take(L.partR));
  float* partP = static_cast<float*>(cv.take(L.partP));
  // recompute what the forward did not save (POET-X section 2.5, checkpointing)
  if (!save_w) {
    st = forward_body(d, x, G_P, G_R, w0, nullptr, U, Vr, W, nullptr, s);
    if (st != POETX_OK) return st;
  } else if (!save_u) {
    POETX_CUDA(launch_gather(x, U, nullptr, d->perm_P, T, n, n, n, es, s), "gather x");
  }
  // B1: dZ = dY[:, p_R]; dW_j = dZ_j G_R,j; dG_R,j = dZ_j^T W_j
  POETX_CUDA(launch_gather(dy, dZ, nullptr, d->perm_R, T, m, m, m, es, s), "gather dy");
  if (bf) {
    POETX_CUDA(bf16_blockdiag(dZ, G_R, dW, T, m, b, true, s), "blockdiag G_R^T");
    POETX_CUDA(bf16_block_grad(dZ, W, partR, dG_R, L.ksR, T, m, b, accumulate, s), "dG_R");
    // B2: dV = dW W0'
    POETX_CUDA(w0_gemm(dW, w0, dV, T, n, m, false, s), "W0' gemm (backward)");
    // B3: dU_j = dV_j G_P,j; dG_P,j = dV_j^T U_j; dX[:, p_P[i]] = dU[:, i]
    POETX_CUDA(bf16_blockdiag(dV, G_P, dU, T, n, b, true, s), "blockdiag G_P^T");
    POETX_CUDA(bf16_block_grad(dV, U, partP, dG_P, L.ksP, T, n, b, accumulate, s), "dG_P");
  } else {
    POETX_CUDA(f32_blockdiag((const float*)dZ, (const float*)G_R, (float*)dW, T, m, b, false, s),
               "blockdiag G_R^T");
    POETX_CUDA(f32_block_grad((const float*)dZ, (const float*)W, dG_R, T, m, b, accumulate, s),
               "dG_R");
    SgemmArgs g;
    g.A = (const float*)dW; g.lda = m;
    g.B = (const float*)W0p; g.ldb = n; g.transB = 0;
    g.C = (float*)dV; g.ldc = n;
    g.M = T; g.N = n; g.K = m; g.batch = 1;
    POETX_CUDA(launch_sgemm(g, s), "W0' gemm (backward)");
    POETX_CUDA(f32_blockdiag((const float*)dV, (const float*)G_P, (float*)dU, T, n, b, false, s),
               "blockdiag G_P^T");
    POETX_CUDA(f32_block_grad((const float*)dV, (const float*)U, dG_P, T, n, b, accumulate, s),
               "dG_P");
  }
  POETX_CUDA(launch_gather(dU, dx, nullptr, d->inv_P, T, n, n, n, es, s), "scatter dx");
  return POETX_OK;
}
}  // namespace

extern "C" {

int poetx_linear_fwd(const poetx_linear_desc* d, const void* x, const void* G_P, const void* G_R,
                     const void* W0p, void* y, void* save_u, void* save_w, void* ws,
                     size_t ws_bytes, void* stream) {
  W0Ref w;
  w.bf16 = W0p;
  return linear_fwd_impl(d, x, G_P, G_R, w, y, save_u, save_w, ws, ws_bytes, stream);
}

int poetx_linear_bwd(const poetx_linear_desc* d, const void* x, const void* dy, const void* G_P,
                     const void* G_R, const void* W0p, const void* save_u, const void* save_w,
                     void* dx, float* dG_P, float* dG_R, int accumulate, void* ws,
                     size_t ws_bytes, void* stream) {
  W0Ref w;
  w.bf16 = W0p;
  return linear_bwd_impl(d, x, dy, G_P, G_R, w, save_u, save_w, dx, dG_P, dG_R, accumulate, ws,
                         ws_bytes, stream);
}

size_t poetx_outer_merge_workspace(int32_t m, int32_t n, int dtype) {
  if (m <= 0 || n <= 0 || (dtype != POETX_F32 && dtype != POETX_BF16)) return 0;
  const size_t es = dtype == POETX_BF16 ? 2 : 4;
  return 2 * align_up((size_t)m * n * es) + align_up((size_t)m * 4) + align_up((size_t)n * 4);
}

int poetx_outer_merge(const void* W0p, const void* G_P, const void* G_R, int32_t m, int32_t n,
                      int32_t b, const int32_t* inv_P, const int32_t* inv_R,
                      const int32_t* perm_P_new, const int32_t* perm_R_new, void* W0p_new,
                      int dtype, void* ws, size_t ws_bytes, void* stream) {
  if (dtype != POETX_F32 && dtype != POETX_BF16) return fail(POETX_ERR_DTYPE, "bad dtype");
  if (m <= 0 || n <= 0 || b <= 0) return fail(POETX_ERR_INVALID_ARG, "sizes must be positive");
  if (m % b != 0 || n % b != 0) return fail(POETX_ERR_SHAPE, "m and n must be multiples of b");
  if (dtype == POETX_BF16 && b % 128 != 0)
    return fail(POETX_ERR_SHAPE, "bf16 outer merge needs b % 128 == 0");
  if (!W0p || !G_P || !G_R || !inv_P || !inv_R || !perm_P_new || !perm_R_new || !W0p_new || !ws)
    return fail(POETX_ERR_INVALID_ARG, "null pointer");
  if (W0p == W0p_new) return fail(POETX_ERR_INVALID_ARG, "W0p and W0p_new must be distinct");
  for (const void* q : {W0p, G_P, G_R, (const void*)inv_P, (const void*)inv_R,
                        (const void*)perm_P_new, (const void*)perm_R_new, (const void*)W0p_new,
                        (const void*)ws})
    if (!aligned16(q)) return fail(POETX_ERR_ALIGN, "pointers must be 16-byte aligned");
  if (ws_bytes < poetx_outer_merge_workspace(m, n, dtype))
    return fail(POETX_ERR_WORKSPACE, "workspace too small");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t es = dtype == POETX_BF16 ? 2 : 4;
  Carve cv(ws);
  void* M1 = cv.take((size_t)m * n * es);
  void* M = cv.take((size_t)m * n * es);
  int32_t* rmap = static_cast<int32_t*>(cv.take((size_t)m * 4));
  int32_t* cmap = static_cast<int32_t*>(cv.take((size_t)n * 4));
  // index maps of the re-merge: W0p_new[i, j] = M[inv_R[perm_R_new[i]], inv_P[perm_P_new[j]]]
  POETX_CUDA(launch_compose_perm(inv_R, perm_R_new, rmap, m, s), "outer merge row map");
  POETX_CUDA(launch_compose_perm(inv_P, perm_P_new, cmap, n, s), "outer merge column map");
  const int nR = m / b;
  if (dtype == POETX_BF16) {
    // M1 rows of block i = G_R,i W0'[rows of block i]: D = A B^T with A[r][k] = G_R,i[r][k]
    // (K-major) and B[c][k] = W0'[ib + k][c] (MN-major)
    UmmaGemm g;
    g.A.ptr = G_R; g.A.rows = (int64_t)nR * b; g.A.cols = b; g.A.ld = b;
    g.A.mn_major = 0; g.A.boff_mn = b;
    g.B.ptr = W0p; g.B.rows = m; g.B.cols = n; g.B.ld = n;
    g.B.mn_major = 1; g.B.boff_k = b;
    g.M = b; g.N = n; g.K = b; g.batch = nR;
    g.D = M1; g.out_f32 = 0; g.ldd = n; g.d_boff = (int64_t)b * n;
    POETX_CUDA(launch_umma_gemm(g, "gemm_blockdiag", s), "outer merge G_R W0'");
    // M[:, block j] = M1[:, block j] G_P,j
    POETX_CUDA(bf16_blockdiag(M1, G_P, M, m, n, b, true, s), "outer merge M1 G_P");
  } else {
    SgemmArgs g;
    g.A = static_cast<const float*>(G_R); g.lda = b; g.sA = (int64_t)b * b;
    g.B = static_cast<const float*>(W0p); g.ldb = n; g.sB = (int64_t)b * n;
    g.C = static_cast<float*>(M1); g.ldc = n; g.sC = (int64_t)b * n;
    g.M = b; g.N = n; g.K = b; g.batch = nR;
    POETX_CUDA(launch_sgemm(g, s), "outer merge G_R W0'");
    POETX_CUDA(f32_blockdiag(static_cast<const float*>(M1), static_cast<const float*>(G_P),
                             static_cast<float*>(M), m, n, b, false, s),
               "outer merge M1 G_P");
  }
  POETX_CUDA(launch_gather(M, W0p_new, rmap, cmap, m, n, n, n, (int)es, s), "outer merge gather");
  return POETX_OK;
}

int poetx_quantize_rows(const void* W, int8_t* q, float* scales, int32_t m, int32_t n, int dtype,
                        void* stream) {
  if (dtype != POETX_F32 && dtype != POETX_BF16) return fail(POETX_ERR_DTYPE, "bad dtype");
  if (m < 0 || n < 0) return fail(POETX_ERR_INVALID_ARG, "negative size");
  if (m == 0 || n == 0) return POETX_OK;
  if (!W || !q || !scales) return fail(POETX_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(W) || !aligned16(q) || !aligned16(scales))
    return fail(POETX_ERR_ALIGN, "pointers must be 16-byte aligned");
  POETX_CUDA(launch_quantize_rows(W, q, scales, m, n, dtype == POETX_BF16 ? 2 : 4,
                                  static_cast<cudaStream_t>(stream)),
             "quantize rows");
  return POETX_OK;
}

int poetx_merge_perm_q8(const void* W0, int8_t* W0q, float* scales, int32_t m, int32_t n,
                        const int32_t* perm_R, const int32_t* perm_P, int dtype, void* stream) {
  if (dtype != POETX_F32 && dtype != POETX_BF16) return fail(POETX_ERR_DTYPE, "bad dtype");
  if (m < 0 || n < 0) return fail(POETX_ERR_INVALID_ARG, "negative size");
  if (m == 0 || n == 0) return POETX_OK;
  if (!W0 || !W0q || !scales || !perm_R || !perm_P)
    return fail(POETX_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(W0) || !aligned16(W0q) || !aligned16(scales) || !aligned16(perm_R) ||
      !aligned16(perm_P))
    return fail(POETX_ERR_ALIGN, "pointers must be 16-byte aligned");
  const int es = dtype == POETX_BF16 ? 2 : 4;
  if ((size_t)n * es > 200 * 1024)
    return fail(POETX_ERR_SHAPE, "rows wider than 200 KB are not supported");
  POETX_CUDA(launch_merge_quantize(W0, perm_R, perm_P, W0q, scales, m, n, es,
                                   static_cast<cudaStream_t>(stream)),
             "merge + quantize");
  return POETX_OK;
}

size_t poetx_linear_q8_scratch(const poetx_linear_desc* d) {
  if (!d || d->dtype != POETX_BF16 || d->m <= 0 || d->n <= 0) return 0;
  return q8_layout(d).total;
}

}  // extern "C"

namespace {
// validates the int8 weight arguments and carves the panel buffer from the front of ws; the
// rest of ws is the layer call's own scratch
int q8_weight(const poetx_linear_desc* d, const int8_t* W0q, const float* scales, void* ws,
              size_t ws_bytes, W0Ref* w, void** rest, size_t* rest_bytes) {
  int st = linear_validate(d);
  if (st != POETX_OK) return st;
  if (d->dtype != POETX_BF16) return fail(POETX_ERR_DTYPE, "int8 base weight needs bf16");
  if (!W0q || !scales) return fail(POETX_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(W0q) || !aligned16(scales) || !aligned16(ws))
    return fail(POETX_ERR_ALIGN, "pointers must be 16-byte aligned");
  const Q8Layout L = q8_layout(d);
  if (!ws || ws_bytes < L.total) return fail(POETX_ERR_WORKSPACE, "scratch too small");
  Carve cv(ws);
  w->q = W0q;
  w->s = scales;
  w->panel = cv.take(L.panel_bytes);
  w->panel_f = L.panel_f;
  w->panel_b = L.panel_b;
  *rest = static_cast<char*>(ws) + L.total;
  *rest_bytes = ws_bytes - L.total;
  return POETX_OK;
}
}  // namespace

extern "C" {

int poetx_linear_fwd_q8(const poetx_linear_desc* d, const void* x, const void* G_P,
                        const void* G_R, const int8_t* W0q, const float* scales, void* y,
                        void* save_u, void* save_w, void* ws, size_t ws_bytes, void* stream) {
  W0Ref w;
  void* rest = nullptr;
  size_t rest_bytes = 0;
  int st = q8_weight(d, W0q, scales, ws, ws_bytes, &w, &rest, &rest_bytes);
  if (st != POETX_OK) return st;
  return linear_fwd_impl(d, x, G_P, G_R, w, y, save_u, save_w, rest, rest_bytes, stream);
}

int poetx_linear_bwd_q8(const poetx_linear_desc* d, const void* x, const void* dy,
                        const void* G_P, const void* G_R, const int8_t* W0q, const float* scales,
                        const void* save_u, const void* save_w, void* dx, float* dG_P,
                        float* dG_R, int accumulate, void* ws, size_t ws_bytes, void* stream) {
  W0Ref w;
  void* rest = nullptr;
  size_t rest_bytes = 0;
  int st = q8_weight(d, W0q, scales, ws, ws_bytes, &w, &rest, &rest_bytes);
  if (st != POETX_OK) return st;
  return linear_bwd_impl(d, x, dy, G_P, G_R, w, save_u, save_w, dx, dG_P, dG_R, accumulate, rest,
                         rest_bytes, stream);
}

int poetx_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  int* flag = device_error_flag();
  if (!flag) return fail(POETX_ERR_CUDA, "device error flag unavailable");
  int v = 0;
  e = cudaMemcpy(&v, flag, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read device flag");
  if (v != 0) {
    const int zero = 0;
    cudaMemcpy(flag, &zero, sizeof(int), cudaMemcpyHostToDevice);
    return fail(v, "a kernel's bounded wait timed out");
  }
  return POETX_OK;
}

uint64_t poetx_launch_count(void) { return g_launches.load(); }

int poetx_profile_begin(const char* name) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (!name || !*name) {
    g_prof_on = false;
    return POETX_OK;
  }
  if (g_ev_start.empty()) {
    g_ev_start.resize(kEventPairs);
    g_ev_stop.resize(kEventPairs);
    for (int i = 0; i < kEventPairs; ++i) {
      cudaError_t e1 = cudaEventCreate(&g_ev_start[i]);
      cudaError_t e2 = cudaEventCreate(&g_ev_stop[i]);
      if (e1 != cudaSuccess || e2 != cudaSuccess) {
        g_ev_start.clear();
        g_ev_stop.clear();
        return cuda_fail(e1 != cudaSuccess ? e1 : e2, "event create");
      }
    }
  }
  g_prof_family = name;
  g_prof_used = 0;
  g_prof_on = true;
  return POETX_OK;
}

int poetx_profile_end(int32_t* launches, double* total_ms) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = false;
  double tot = 0.0;
  for (int i = 0; i < g_prof_used; ++i) {
    cudaError_t e = cudaEventSynchronize(g_ev_stop[i]);
    if (e != cudaSuccess) return cuda_fail(e, "event synchronize");
    float ms = 0.f;
    e = cudaEventElapsedTime(&ms, g_ev_start[i], g_ev_stop[i]);
    if (e != cudaSuccess) return cuda_fail(e, "event elapsed");
    tot += ms;
  }
  if (launches) *launches = g_prof_used;
  if (total_ms) *total_ms = tot;
  return POETX_OK;
}

}  // extern "C"
