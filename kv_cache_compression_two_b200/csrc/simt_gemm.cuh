// simt_gemm.cuh -- register-tiled GEMM on the fp32 CUDA cores.
//
// acc[m][n] = sum_k opA(m, k) * opB(k, n), handed element by element to an
// epilogue functor.  64 x 64 output tile per CTA, 256 threads with a 4 x 4
// micro-tile each (rows ty + 16 i, columns tx + 16 j, so shared-memory reads
// are broadcast or conflict-free), K staged 16 at a time.  Used where fp32 (or
// fp64-accumulated) accuracy is required: the blocked Cholesky's trailing
// updates and triangular-solve updates, the refinement residual, the
// G dW product of epsilon, and the fp32 statistics path.
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
