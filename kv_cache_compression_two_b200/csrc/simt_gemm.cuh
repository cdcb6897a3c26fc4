// simt_gemm.cuh -- register-tiled GEMM on the fp32 CUDA cores.
//
// acc[m][n] = sum_k opA(m, k) * opB(k, n), handed element by element to an
// epilogue functor.  64 x 64 output tile per CTA, 256 threads with a 4 x 4
// micro-tile each (rows ty + 16 i, columns tx + 16 j, so shared-memory reads
// are broadcast or conflict-free), K staged 16 at a time.  Used where fp32 (or
// fp64-accumulated) accuracy is required: the refinement residual, the
// G dW product of epsilon and the fp32 statistics path.
#pragma once

#include "common.cuh"

namespace ispa {

// Operand views.  Plain: element (r, c) = p[r * ld + c] (or transposed).
// Symmetric-from-upper: element (r, c) = p[min(r,c) * ld + max(r,c)].
// Difference: element = p[...] - p2[...].
enum OperandKind { OP_N = 0, OP_T = 1, OP_SYM_UPPER = 2 };

struct Operand {
  const float *p;
  const float *p2;  // optional subtrahend (same layout), nullptr if unused
  long long ld;
};

template <int KIND>
__device__ __forceinline__ float op_load(const Operand &o, int r, int c) {
  long long off;
  if (KIND == OP_N)
    off = (long long)r * o.ld + c;
  else if (KIND == OP_T)
    off = (long long)c * o.ld + r;
  else
    off = r <= c ? (long long)r * o.ld + c : (long long)c * o.ld + r;
  float x = o.p[off];
  if (o.p2) x -= o.p2[off];
  return x;
}

// Tile filter: 0 = every tile, 1 = tiles touching i >= j, 2 = tiles touching i <= j.
template <int KA, int KB, typename Acc, int TRI, class Epi>
__global__ void __launch_bounds__(256) simt_gemm_kernel(int M, int N, int K, Operand A, Operand B, Epi epi) {
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  if (TRI == 1 && n0 > m0 + 63) return;
  if (TRI == 2 && m0 > n0 + 63) return;
  __shared__ float As[16][64];
  __shared__ float Bs[16][64];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  Acc acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = Acc(0);
  for (int k0 = 0; k0 < K; k0 += 16) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int idx = tid + 256 * e;  // 0..1023
      // A tile: 64 rows x 16 k; B tile: 16 k x 64 cols
      const int ar = idx >> 4, ak = idx & 15;
      const int gm = m0 + ar, gk = k0 + ak;
      As[ak][ar] = (gm < M && gk < K) ? op_load<KA>(A, gm, gk) : 0.f;
      const int bk = idx >> 6, bc = idx & 63;
      const int gk2 = k0 + bk, gn = n0 + bc;
      Bs[bk][bc] = (gk2 < K && gn < N) ? op_load<KB>(B, gk2, gn) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      Acc a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = Acc(As[kk][ty + 16 * i]);
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Acc(Bs[kk][tx + 16 * j]);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  epi.begin();
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = m0 + ty + 16 * i, n = n0 + tx + 16 * j;
      if (m < M && n < N) epi(m, n, acc[i][j]);
    }
  epi.end();
}

template <int KA, int KB, typename Acc, int TRI, class Epi>
inline cudaError_t simt_gemm(int M, int N, int K, Operand A, Operand B, Epi epi, cudaStream_t s) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  dim3 grid((N + 63) / 64, (M + 63) / 64);
  simt_gemm_kernel<KA, KB, Acc, TRI, Epi><<<grid, 256, 0, s>>>(M, N, K, A, B, epi);
  note_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Larger-tile variant for big row-major products C = A[M,K] B[K,N] (both
// operands plain row-major, lda/ldb multiples of 4, 16-byte aligned bases):
// 128 x 128 output tile, 256 threads with 8 x 8 accumulators each (two 4 x 4
// quadrants 64 apart in each dimension, so shared-memory reads are float4 and
// conflict-free), K staged 8 at a time through double-buffered shared memory
// with the next stage prefetched into registers.  Grid z-slice z covers the
// K range [z kchunk, (z + 1) kchunk) (kchunk a multiple of 8), so the epilogue
// sees partial sums when gridDim.z > 1; with upper != 0 only tiles that reach
// the upper triangle (some m <= n) run.
// ---------------------------------------------------------------------------
template <class Epi>
__global__ void __launch_bounds__(256) simt_gemm_nn128_kernel(int M, int N, int K, const float *__restrict__ A,
                                                              long long lda, const float *__restrict__ B,
                                                              long long ldb, Epi epi, int kchunk, int upper) {
  __shared__ __align__(16) float As[2][8][128];
  __shared__ __align__(16) float Bs[2][8][128];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * 128, n0 = blockIdx.x * 128;
  if (upper && m0 > n0 + 127) return;
  const int k_lo = blockIdx.z * kchunk, k_hi = min(K, k_lo + kchunk);
  if (k_lo >= k_hi) return;
  // A tile 128 x 8: thread loads row (tid >> 1), 4 k values at (tid & 1) * 4
  const int a_row = tid >> 1, a_k = (tid & 1) * 4;
  // B tile 8 x 128: thread loads k row (tid >> 5), 4 columns at (tid & 31) * 4
  const int b_k = tid >> 5, b_col = (tid & 31) * 4;
  auto load_a = [&](int k0, float4 &v) {
    const int gm = m0 + a_row, gk = k0 + a_k;
    if (gm < M && gk + 3 < k_hi) {
      v = *reinterpret_cast<const float4 *>(A + (long long)gm * lda + gk);
    } else {
      float t[4];
      for (int i = 0; i < 4; ++i) t[i] = (gm < M && gk + i < k_hi) ? A[(long long)gm * lda + gk + i] : 0.f;
      v = make_float4(t[0], t[1], t[2], t[3]);
    }
  };
  auto load_b = [&](int k0, float4 &v) {
    const int gk = k0 + b_k, gn = n0 + b_col;
    if (gk < k_hi && gn + 3 < N) {
      v = *reinterpret_cast<const float4 *>(B + (long long)gk * ldb + gn);
    } else {
      float t[4];
      for (int i = 0; i < 4; ++i) t[i] = (gk < k_hi && gn + i < N) ? B[(long long)gk * ldb + gn + i] : 0.f;
      v = make_float4(t[0], t[1], t[2], t[3]);
    }
  };
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  float4 ra, rb;
  load_a(k_lo, ra);
  load_b(k_lo, rb);
  int buf = 0;
  As[0][a_k + 0][a_row] = ra.x;
  As[0][a_k + 1][a_row] = ra.y;
  As[0][a_k + 2][a_row] = ra.z;
  As[0][a_k + 3][a_row] = ra.w;
  *reinterpret_cast<float4 *>(&Bs[0][b_k][b_col]) = rb;
  __syncthreads();
  for (int k0 = k_lo; k0 < k_hi; k0 += 8) {
    const bool more = k0 + 8 < k_hi;
    if (more) {
      load_a(k0 + 8, ra);
      load_b(k0 + 8, rb);
    }
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4 *>(&As[buf][kk][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4 *>(&As[buf][kk][ty * 4 + 64]);
      const float4 b0 = *reinterpret_cast<const float4 *>(&Bs[buf][kk][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4 *>(&Bs[buf][kk][tx * 4 + 64]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    if (more) {
      const int nb = buf ^ 1;
      As[nb][a_k + 0][a_row] = ra.x;
      As[nb][a_k + 1][a_row] = ra.y;
      As[nb][a_k + 2][a_row] = ra.z;
      As[nb][a_k + 3][a_row] = ra.w;
      *reinterpret_cast<float4 *>(&Bs[nb][b_k][b_col]) = rb;
      __syncthreads();
      buf = nb;
    }
  }
  epi.begin();
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int m = m0 + ty * 4 + (i & 3) + (i >> 2) * 64, n = n0 + tx * 4 + (j & 3) + (j >> 2) * 64;
      if (m < M && n < N) epi(m, n, acc[i][j]);
    }
  epi.end();
}

template <class Epi>
inline cudaError_t simt_gemm_nn128(int M, int N, int K, const float *A, long long lda, const float *B, long long ldb,
                                   Epi epi, cudaStream_t s, int nsplit = 1, int upper = 0) {
  if (M <= 0 || N <= 0 || K <= 0) return cudaSuccess;
  const int kchunk = ((K + nsplit - 1) / nsplit + 7) / 8 * 8;
  dim3 grid((N + 127) / 128, (M + 127) / 128, (K + kchunk - 1) / kchunk);
  simt_gemm_nn128_kernel<Epi><<<grid, 256, 0, s>>>(M, N, K, A, lda, B, ldb, epi, kchunk, upper);
  note_launch();
  return cudaGetLastError();
}

// ---- common epilogues ----
// out[m*ld + n] = beta * out[...] + alpha * acc   (restricted by `tri`: 0 all, 1 m>=n, 2 m<=n)
struct EpiAxpby {
  float *out;
  long long ld;
  float alpha, beta;
  int tri;
  __device__ void begin() {}
  __device__ void end() {}
  template <typename Acc>
  __device__ void operator()(int m, int n, Acc acc) {
    if ((tri == 1 && m < n) || (tri == 2 && m > n)) return;
    float *p = out + (long long)m * ld + n;
    *p = (beta == 0.f ? 0.f : beta * *p) + alpha * (float)acc;
  }
};

}  // namespace ispa
