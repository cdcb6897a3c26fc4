// ridge.cu -- closed-form absorption: dW = (G + lambda I)^-1 C and epsilon.
//
// Blocked right-looking Cholesky in fp32 (block NB = 64):
//   for each diagonal block k:  factor L_kk and invert it (one CTA, shared memory),
//                               L_ik = A_ik Linv_kk^T for the rows below (SIMT GEMM),
//                               A_ij -= L_ik L_jk^T on the trailing lower triangle (SIMT GEMM).
// then the blocked forward and backward substitutions on the Dout right-hand
// sides (diagonal blocks applied as GEMMs with Linv_kk), optional iterative
// refinement with residuals accumulated in fp64, and
// epsilon = r2 - 2<dW, C> + <dW, G dW> with fp64 reductions.
#include <mutex>

#include "internal.h"
#include "simt_gemm.cuh"

namespace ispa {

namespace {

constexpr int NB = 64;

struct Ws {
  float *L;      // [D, D] lower Cholesky factor (working copy)
  float *Linv;   // [ceil(D / 64), 64, 64] inverses of the diagonal blocks of L
  float *Rres;   // [D, Dout] refinement residual / correction
  double *acc;   // [0] <dW, C>  [1] <dW, G dW>  [2] trace(G)  [3] lambda_eff
  int *flag;     // non-zero once a pivot failed
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

Ws carve(void *base, int D, int Dout) {
  char *p = static_cast<char *>(base);
  Ws w;
  w.L = reinterpret_cast<float *>(p);
  p += align256((size_t)D * D * sizeof(float));
  w.Linv = reinterpret_cast<float *>(p);
  p += align256((size_t)((D + NB - 1) / NB) * NB * NB * sizeof(float));
  w.Rres = reinterpret_cast<float *>(p);
  p += align256((size_t)D * Dout * sizeof(float));
  w.acc = reinterpret_cast<double *>(p);
  p += 64;
  w.flag = reinterpret_cast<int *>(p);
  return w;
}

__global__ void trace_kernel(int D, const float *__restrict__ G, double *acc) {
  double s = 0.0;
  for (int i = threadIdx.x; i < D; i += blockDim.x) s += (double)G[(long long)i * D + i];
  s = warp_sum_d(s);
  __shared__ double part[32];
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += part[w];
    acc[2] = t;
  }
}

__global__ void init_kernel(int D, int Dout, const float *__restrict__ G, const float *__restrict__ C,
                            float lambda, int relative, Ws w, float *dW) {
  const double lam = relative ? (double)lambda * w.acc[2] / D : (double)lambda;
  const float lamf = (float)lam;
  const long long nDD = (long long)D * D, nDO = (long long)D * Dout;
  const long long stride = (long long)gridDim.x * blockDim.x;
  const long long t0 = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (t0 == 0) {
    w.acc[0] = 0.0;
    w.acc[1] = 0.0;
    w.acc[3] = (double)lamf;
    *w.flag = 0;
  }
  for (long long e = t0; e < nDD; e += stride) {
    const int i = (int)(e / D), j = (int)(e - (long long)i * D);
    float x = 0.f;
    if (i >= j) x = G[(long long)j * D + i] + (i == j ? lamf : 0.f);
    w.L[e] = x;
  }
  for (long long e = t0; e < nDO; e += stride) dW[e] = C[e];
}

// Factors the nb x nb diagonal block at kb0 in place (nb <= 64) and writes the
// inverse of its lower factor, padded to 64 x 64 with the identity, to Linv.
// One CTA of 512 threads: per column one pivot, a scaled column and a rank-1
// update of the trailing triangle spread over all threads; the inverse is
// formed row by row (X = L^-1 solves L X = I), each row's entries in parallel.
__global__ void __launch_bounds__(512) potrf_inv_kernel(int D, int kb0, float *L, float *Linv, int *flag,
                                                        DevErr err) {
  __shared__ float A[NB][NB + 1];
  __shared__ float X[NB][NB + 1];
  const int nb = min(NB, D - kb0);
  const int t = threadIdx.x;
  for (int e = t; e < NB * NB; e += blockDim.x) {
    const int r = e / NB, c = e % NB;
    A[r][c] = (r < nb && c < nb) ? L[(long long)(kb0 + r) * D + kb0 + c] : (r == c ? 1.f : 0.f);
  }
  __syncthreads();
  for (int c = 0; c < NB; ++c) {
    if (t == 0) {
      float piv = A[c][c];
      if (!(piv > 0.f)) {
        if (atomicExch(flag, 1) == 0) report_error(err, ISPA_ERR_NOT_SPD, kb0 + c + 1);
        piv = __int_as_float(0x7fc00000);
      }
      A[c][c] = sqrtf(piv);
    }
    __syncthreads();
    const float inv_d = 1.f / A[c][c];
    if (t > c && t < NB) A[t][c] *= inv_d;
    __syncthreads();
    // rank-1 update of the trailing lower triangle: 8 threads per row i = t / 8,
    // each taking the columns j = c+1+q, c+9+q, ... (q = t % 8) up to i
    {
      const int i = t >> 3, q = t & 7;
      if (i > c) {
        const float lic = A[i][c];
        for (int j = c + 1 + q; j <= i; j += 8) A[i][j] -= lic * A[j][c];
      }
    }
    __syncthreads();
  }
  // X = L^-1 (lower), row by row: X[r][j] = (delta_rj - sum_{j<=p<r} L[r][p] X[p][j]) / L[r][r].
  // 8 threads share one entry j = t / 8 (partial sums over p = q, q+8, ...), combined by shuffles.
  {
    const int j = t >> 3, q = t & 7;
    for (int r = 0; r < NB; ++r) {
      float s = 0.f;
      if (j <= r)
        for (int p = j + q; p < r; p += 8) s += A[r][p] * X[p][j];
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      s += __shfl_xor_sync(0xffffffffu, s, 4);
      if (q == 0) X[r][j] = (j <= r) ? (((j == r) ? 1.f : 0.f) - s) / A[r][r] : 0.f;
      __syncthreads();
    }
  }
  for (int e = t; e < NB * NB; e += blockDim.x) {
    const int r = e / NB, c = e % NB;
    Linv[e] = X[r][c];
    if (r < nb && c <= r) L[(long long)(kb0 + r) * D + kb0 + c] = A[r][c];
  }
}

// Rres = C - (G + lambda I) X, accumulated in fp64.
struct EpiResidual {
  float *out;
  const float *C, *X;
  const double *acc;
  int ld;
  __device__ void begin() {}
  __device__ void end() {}
  __device__ void operator()(int m, int n, double a) {
    const long long o = (long long)m * ld + n;
    out[o] = (float)((double)C[o] - a - acc[3] * (double)X[o]);
  }
};

// acc[1] += sum dW[m][n] * (G dW)[m][n]
struct EpiDotG {
  const float *dW;
  double *acc;
  int ld;
  double part;
  __device__ void begin() { part = 0.0; }
  __device__ void operator()(int m, int n, float a) { part += (double)dW[(long long)m * ld + n] * (double)a; }
  __device__ void end() {
    const double s = warp_sum_d(part);
    if ((threadIdx.x & 31) == 0) atomicAdd(acc + 1, s);
  }
};

__global__ void add_kernel(long long n, float *__restrict__ X, const float *__restrict__ dX) {
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x)
    X[e] += dX[e];
}

// out[i][j] = G[min(i,j)][max(i,j)]: the full symmetric matrix from its upper triangle.
__global__ void symmetrize_kernel(int D, const float *__restrict__ G, float *out) {
  const long long n = (long long)D * D;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
    const int i = (int)(e / D), j = (int)(e - (long long)i * D);
    out[e] = i <= j ? G[e] : G[(long long)j * D + i];
  }
}

__global__ void dot_kernel(long long n, const float *__restrict__ a, const float *__restrict__ b, double *out) {
  double s = 0.0;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x)
    s += (double)a[e] * (double)b[e];
  s = warp_sum_d(s);
  if ((threadIdx.x & 31) == 0) atomicAdd(out, s);
}

__global__ void finalize_kernel(long long n, const double *__restrict__ r2, Ws w, float *dW, double *eps) {
  const bool bad = *w.flag != 0;
  if (blockIdx.x == 0 && threadIdx.x == 0)
    *eps = bad ? __longlong_as_double(0x7ff8000000000000LL) : (*r2 - 2.0 * w.acc[0] + w.acc[1]);
  if (!bad) return;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x)
    dW[e] = __int_as_float(0x7fc00000);
}

// Forward then backward blocked substitution on Y [D, Dout] in place, using the
// inverted diagonal blocks: Y_k <- Linv_kk Y_k (a small GEMM whose CTAs each
// read their whole 64-row block column before writing it, so it may run in
// place), then the update of the remaining block rows.
cudaError_t cholesky_solve(int D, int Dout, const float *L, const float *Linv, float *Y, cudaStream_t s) {
  for (int kb0 = 0; kb0 < D; kb0 += NB) {
    const int nb = min(NB, D - kb0);
    const float *Li = Linv + (long long)(kb0 / NB) * NB * NB;
    cudaError_t e = simt_gemm<OP_N, OP_N, float, 0>(nb, Dout, nb, Operand{Li, nullptr, NB},
                                                    Operand{Y + (long long)kb0 * Dout, nullptr, Dout},
                                                    EpiAxpby{Y + (long long)kb0 * Dout, Dout, 1.f, 0.f, 0}, s);
    if (e != cudaSuccess) return e;
    const int below = D - kb0 - nb;
    if (below > 0) {
      e = simt_gemm<OP_N, OP_N, float, 0>(below, Dout, nb, Operand{L + (long long)(kb0 + nb) * D + kb0, nullptr, D},
                                          Operand{Y + (long long)kb0 * Dout, nullptr, Dout},
                                          EpiAxpby{Y + (long long)(kb0 + nb) * Dout, Dout, -1.f, 1.f, 0}, s);
      if (e != cudaSuccess) return e;
    }
  }
  const int last0 = ((D - 1) / NB) * NB;
  for (int kb0 = last0; kb0 >= 0; kb0 -= NB) {
    const int nb = min(NB, D - kb0);
    const float *Li = Linv + (long long)(kb0 / NB) * NB * NB;
    cudaError_t e = simt_gemm<OP_T, OP_N, float, 0>(nb, Dout, nb, Operand{Li, nullptr, NB},
                                                    Operand{Y + (long long)kb0 * Dout, nullptr, Dout},
                                                    EpiAxpby{Y + (long long)kb0 * Dout, Dout, 1.f, 0.f, 0}, s);
    if (e != cudaSuccess) return e;
    if (kb0 > 0) {
      e = simt_gemm<OP_T, OP_N, float, 0>(kb0, Dout, nb, Operand{L + (long long)kb0 * D, nullptr, D},
                                          Operand{Y + (long long)kb0 * Dout, nullptr, Dout},
                                          EpiAxpby{Y, Dout, -1.f, 1.f, 0}, s);
      if (e != cudaSuccess) return e;
    }
  }
  return cudaGetLastError();
}

}  // namespace

size_t ridge_workspace_bytes(int D, int Dout) {
  return align256((size_t)D * D * sizeof(float)) + align256((size_t)((D + NB - 1) / NB) * NB * NB * sizeof(float)) +
         align256((size_t)D * Dout * sizeof(float)) + 256;
}

// ---------------------------------------------------------------------------
// Allocation-free variant (ispa_ridge_solve_noalloc).  Its scratch -- the
// working copy of the Cholesky factor, the refinement residual and a few
// accumulators -- lives in this file-scope device array instead of a
// caller-supplied workspace.  Every device that loads the library holds the
// array until the process exits.  Host code must not pass the symbol itself to
// a kernel (on the host it only names a host-side shadow); the device address
// is looked up once per device with cudaGetSymbolAddress.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = (size_t)ISPA_RIDGE_NOALLOC_MAX_D * ISPA_RIDGE_NOALLOC_MAX_D * 4 +
                                        (size_t)ISPA_RIDGE_NOALLOC_MAX_D * NB * 4 +
                                        (size_t)ISPA_RIDGE_NOALLOC_MAX_D * ISPA_RIDGE_NOALLOC_MAX_DOUT * 4 + 256;
static __device__ __align__(256) unsigned char g_ridge_scratch[kNoAllocScratchBytes];

ispa_status ridge_noalloc_scratch(void **out) {
  static std::mutex mu;
  static void *addr[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(ISPA_ERR_CUDA, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_ridge_scratch);
    if (e != cudaSuccess) return cuda_status(e, "cudaGetSymbolAddress(ridge scratch)");
    addr[dev] = p;
  }
  *out = addr[dev];
  static_assert(ISPA_RIDGE_NOALLOC_MAX_D % NB == 0 && ISPA_RIDGE_NOALLOC_MAX_D % 64 == 0,
                "the largest workspace must fit the scratch exactly");
  return ISPA_OK;
}

ispa_status launch_ridge(int D, int Dout, const float *G, const float *C, const double *r2, float lambda,
                         int lambda_relative, int refine_steps, float *dW, double *eps, void *ws_base,
                         cudaStream_t s) {
  DevErr err;
  ispa_status st = device_err(&err);
  if (st != ISPA_OK) return st;
  Ws w = carve(ws_base, D, Dout);
  const int grid = sm_count() * 4;
  trace_kernel<<<1, 256, 0, s>>>(D, G, w.acc);
  init_kernel<<<grid, 256, 0, s>>>(D, Dout, G, C, lambda, lambda_relative, w, dW);
  note_launch(2);
  for (int kb0 = 0; kb0 < D; kb0 += NB) {
    float *Li = w.Linv + (long long)(kb0 / NB) * NB * NB;
    potrf_inv_kernel<<<1, 512, 0, s>>>(D, kb0, w.L, Li, w.flag, err);
    note_launch();
    const int below = D - kb0 - NB;
    if (below > 0) {
      // panel: L[i, kb] = A[i, kb] Linv_kk^T for the rows below (in place: each CTA owns whole rows)
      float *panel = w.L + (long long)(kb0 + NB) * D + kb0;
      cudaError_t e = simt_gemm<OP_N, OP_T, float, 0>(below, NB, NB, Operand{panel, nullptr, D},
                                                      Operand{Li, nullptr, NB}, EpiAxpby{panel, D, 1.f, 0.f, 0}, s);
      if (e != cudaSuccess) return cuda_status(e, "ridge panel");
      const int j0 = kb0 + NB;
      e = simt_gemm<OP_N, OP_T, float, 1>(below, below, NB, Operand{w.L + (long long)j0 * D + kb0, nullptr, D},
                                          Operand{w.L + (long long)j0 * D + kb0, nullptr, D},
                                          EpiAxpby{w.L + (long long)j0 * D + j0, D, -1.f, 1.f, 1}, s);
      if (e != cudaSuccess) return cuda_status(e, "ridge trailing update");
    }
  }
  cudaError_t e = cholesky_solve(D, Dout, w.L, w.Linv, dW, s);
  if (e != cudaSuccess) return cuda_status(e, "ridge solve");
  const long long nDO = (long long)D * Dout;
  for (int r = 0; r < refine_steps; ++r) {
    e = simt_gemm<OP_SYM_UPPER, OP_N, double, 0>(D, Dout, D, Operand{G, nullptr, D}, Operand{dW, nullptr, Dout},
                                                 EpiResidual{w.Rres, C, dW, w.acc, Dout}, s);
    if (e != cudaSuccess) return cuda_status(e, "ridge residual");
    e = cholesky_solve(D, Dout, w.L, w.Linv, w.Rres, s);
    if (e != cudaSuccess) return cuda_status(e, "ridge refinement solve");
    add_kernel<<<grid, 256, 0, s>>>(nDO, dW, w.Rres);
    note_launch();
  }
  dot_kernel<<<grid, 256, 0, s>>>(nDO, dW, C, w.acc);
  note_launch();
  if (D % 4 == 0 && Dout % 4 == 0) {
    // the factor is no longer needed: expand G to the full symmetric matrix there
    // so that the G dW product reads both operands row-major with 16-byte loads
    symmetrize_kernel<<<grid, 256, 0, s>>>(D, G, w.L);
    note_launch();
    e = simt_gemm_nn128(D, Dout, D, w.L, D, dW, Dout, EpiDotG{dW, w.acc, Dout, 0.0}, s);
  } else {
    e = simt_gemm<OP_SYM_UPPER, OP_N, float, 0>(D, Dout, D, Operand{G, nullptr, D}, Operand{dW, nullptr, Dout},
                                                EpiDotG{dW, w.acc, Dout, 0.0}, s);
  }
  if (e != cudaSuccess) return cuda_status(e, "ridge G dW");
  finalize_kernel<<<grid, 256, 0, s>>>(nDO, r2, w, dW, eps);
  note_launch();
  return cuda_status(cudaGetLastError(), "ridge launch");
}

}  // namespace ispa
