// simt_gemm_batched.cuh -- batched 128 x 128-tile fp32 GEMM on the CUDA cores
// for the recursive inversion of the Cholesky factor (ridge.cu).
#pragma once

#include "common.cuh"

namespace ispa {

// ---------------------------------------------------------------------------
// Batched 128 x 128-tile GEMM for the triangular products of the recursive
// inversion: C = alpha A B + beta C, A [M, K], B [K, N], all row-major.  One
// z-slice of the grid per job.  A triangle that is zero is skipped at tile
// granularity through the K range of each output tile (the skipped region
// must hold zeros or lie outside the triangle):
//   kTriALower: A[m][k] = 0 for k > m   ->  k <  m0 + 128
//   kTriBLower: B[k][n] = 0 for k < n   ->  k >= n0
// Operands are read with 16-byte loads when every leading dimension is a
// multiple of 4 and every base 16-byte aligned (vec), element by element
// otherwise.  256 threads with 8 x 8 accumulators each (two 4 x 4 quadrants
// 64 apart in each dimension), K staged 8 at a time through double-buffered
// shared memory with the next stage prefetched into registers.
// ---------------------------------------------------------------------------
enum { kTriNone = 0, kTriALower = 1, kTriBLower = 3 };

struct GemmJob {
  const float *A;
  const float *B;
  float *C;
  long long lda, ldb, ldc;
  int M, N, K, tri;
  float alpha, beta;
};

constexpr int kMaxGemmJobs = 32;
struct GemmBatch {
  GemmJob job[kMaxGemmJobs];
};

// Split K: with nsplit > 1, grid z-slice z handles job z / nsplit and the K
// chunk z % nsplit of length kchunk (a multiple of 8) of every output tile's
// K range, and adds alpha times its partial product to C with atomics (C must
// then hold beta C already: zero for beta = 0).
__global__ void __launch_bounds__(256, 2) simt_gemm_batched_kernel(GemmBatch batch, int vec, int nsplit, int kchunk) {
  const GemmJob &j = batch.job[blockIdx.z / nsplit];
  const int chunk = blockIdx.z % nsplit;
  const int m0 = blockIdx.y * 128, n0 = blockIdx.x * 128;
  if (m0 >= j.M || n0 >= j.N) return;
  int k_lo = 0, k_hi = j.K;
  if (j.tri == kTriALower) k_hi = min(j.K, m0 + 128);
  if (j.tri == kTriBLower) k_lo = n0;
  if (nsplit > 1) {
    k_lo += chunk * kchunk;
    k_hi = min(k_hi, k_lo + kchunk);
    if (k_lo >= k_hi) return;
  }
  __shared__ __align__(16) float As[2][8][128];
  __shared__ __align__(16) float Bs[2][8][128];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  // A tile 128 (m) x 8 (k): thread takes row tid / 2, 4 k at (tid & 1) * 4
  // B tile 8 (k) x 128 (n): thread takes k row tid / 32, 4 columns at (tid & 31) * 4
  const int a_r = tid >> 1, a_c = (tid & 1) * 4;
  const int b_k = tid >> 5, b_col = (tid & 31) * 4;
  auto load_a = [&](int k0, float (&v)[4]) {
    const int gm = m0 + a_r, gk = k0 + a_c;
    if (vec && gm < j.M && gk + 3 < k_hi) {
      const float4 t = *reinterpret_cast<const float4 *>(j.A + (long long)gm * j.lda + gk);
      v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    } else {
      for (int i = 0; i < 4; ++i) v[i] = (gm < j.M && gk + i < k_hi) ? j.A[(long long)gm * j.lda + gk + i] : 0.f;
    }
  };
  auto load_b = [&](int k0, float (&v)[4]) {
    const int gk = k0 + b_k, gn = n0 + b_col;
    if (vec && gk < k_hi && gn + 3 < j.N) {
      const float4 t = *reinterpret_cast<const float4 *>(j.B + (long long)gk * j.ldb + gn);
      v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    } else {
      for (int i = 0; i < 4; ++i) v[i] = (gk < k_hi && gn + i < j.N) ? j.B[(long long)gk * j.ldb + gn + i] : 0.f;
    }
  };
  auto stage = [&](int buf, const float (&ra)[4], const float (&rb)[4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) As[buf][a_c + i][a_r] = ra[i];
    *reinterpret_cast<float4 *>(&Bs[buf][b_k][b_col]) = make_float4(rb[0], rb[1], rb[2], rb[3]);
  };
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[i][c] = 0.f;
  float ra[4], rb[4];
  load_a(k_lo, ra);
  load_b(k_lo, rb);
  int buf = 0;
  stage(0, ra, rb);
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
        for (int c = 0; c < 8; ++c) acc[i][c] = fmaf(a[i], b[c], acc[i][c]);
    }
    if (more) {
      stage(buf ^ 1, ra, rb);
      __syncthreads();
      buf ^= 1;
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int m = m0 + ty * 4 + (i & 3) + (i >> 2) * 64, n = n0 + tx * 4 + (c & 3) + (c >> 2) * 64;
      if (m < j.M && n < j.N) {
        float *p = j.C + (long long)m * j.ldc + n;
        if (nsplit > 1)
          atomicAdd(p, j.alpha * acc[i][c]);
        else
          *p = j.alpha * acc[i][c] + (j.beta == 0.f ? 0.f : j.beta * *p);
      }
    }
}

}  // namespace ispa

namespace ispa {

// ---------------------------------------------------------------------------
// Pipelined form of simt_gemm_batched_kernel (same jobs, triangles and split
// K), for 16-byte-aligned operands with leading dimensions that are multiples
// of 4: K advances 16 at a time through a kPipeStages-deep cp.async ring, so
// the L2 latency of a stage hides behind the arithmetic of the stages ahead.
// B is copied as it is ([k][n]); A is kept as [m][k] (row stride kPipeALd)
// and read as broadcast scalars.  Edges are zero-filled by the copy
// (src-size < 16).
// ---------------------------------------------------------------------------
constexpr int kPipeStages = 4, kPipeBK = 16, kPipeALd = 20;
constexpr int kPipeStageFloats = 128 * kPipeALd + kPipeBK * 128;  // A + B
constexpr size_t kPipeSmemBytes = sizeof(float) * kPipeStages * kPipeStageFloats;

__device__ __forceinline__ void cp_async16_zfill(void *dst, const void *src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}

__global__ void __launch_bounds__(256, 2) simt_gemm_pipe_kernel(GemmBatch batch, int nsplit, int kchunk) {
  extern __shared__ __align__(16) float pipe_smem[];
  const GemmJob &j = batch.job[blockIdx.z / nsplit];
  const int chunk = blockIdx.z % nsplit;
  const int m0 = blockIdx.y * 128, n0 = blockIdx.x * 128;
  if (m0 >= j.M || n0 >= j.N) return;
  int k_lo = 0, k_hi = j.K;
  if (j.tri == kTriALower) k_hi = min(j.K, m0 + 128);
  if (j.tri == kTriBLower) k_lo = n0;
  if (nsplit > 1) {
    k_lo += chunk * kchunk;
    k_hi = min(k_hi, k_lo + kchunk);
  }
  if (k_lo >= k_hi) {
    if (nsplit > 1) return;  // nothing to add
  }
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int nk = k_hi > k_lo ? (k_hi - k_lo + kPipeBK - 1) / kPipeBK : 0;

  auto issue = [&](int kb) {
    float *As = pipe_smem + (kb % kPipeStages) * kPipeStageFloats;
    float *Bs = As + 128 * kPipeALd;
    const int k0 = k_lo + kb * kPipeBK;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int e = tid + 256 * u;
      {  // B: 16 rows x 32 chunks of 4 columns
        const int r = e >> 5, c = (e & 31) * 4, gk = k0 + r, gn = n0 + c;
        const int nv = (gk < k_hi) ? max(0, min(4, j.N - gn)) : 0;
        cp_async16_zfill(Bs + r * 128 + c, nv ? j.B + (long long)gk * j.ldb + gn : j.B, nv * 4);
      }
      {  // A: 128 rows (m) x 4 chunks of 4 k
        const int r = e >> 2, c = (e & 3) * 4, gm = m0 + r, gk = k0 + c;
        const int nv = (gm < j.M) ? max(0, min(4, k_hi - gk)) : 0;
        cp_async16_zfill(As + r * kPipeALd + c, nv ? j.A + (long long)gm * j.lda + gk : j.A, nv * 4);
      }
    }
  };

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[i][c] = 0.f;
#pragma unroll
  for (int s = 0; s < kPipeStages - 1; ++s) {
    if (s < nk) issue(s);
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  for (int kb = 0; kb < nk; ++kb) {
    asm volatile("cp.async.wait_group %0;" ::"n"(kPipeStages - 2) : "memory");
    __syncthreads();  // stage kb landed for every thread; stage kb - 1 is free
    if (kb + kPipeStages - 1 < nk) issue(kb + kPipeStages - 1);
    asm volatile("cp.async.commit_group;" ::: "memory");
    const float *As = pipe_smem + (kb % kPipeStages) * kPipeStageFloats;
    const float *Bs = As + 128 * kPipeALd;
#pragma unroll
    for (int kk = 0; kk < kPipeBK; ++kk) {
      float a[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[(ty * 4 + i) * kPipeALd + kk];
        a[4 + i] = As[(ty * 4 + 64 + i) * kPipeALd + kk];
      }
      const float4 b0 = *reinterpret_cast<const float4 *>(Bs + kk * 128 + tx * 4);
      const float4 b1 = *reinterpret_cast<const float4 *>(Bs + kk * 128 + tx * 4 + 64);
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[i][c] = fmaf(a[i], b[c], acc[i][c]);
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int m = m0 + ty * 4 + (i & 3) + (i >> 2) * 64, n = n0 + tx * 4 + (c & 3) + (c >> 2) * 64;
      if (m < j.M && n < j.N) {
        float *p = j.C + (long long)m * j.ldc + n;
        if (nsplit > 1)
          atomicAdd(p, j.alpha * acc[i][c]);
        else
          *p = j.alpha * acc[i][c] + (j.beta == 0.f ? 0.f : j.beta * *p);
      }
    }
}

}  // namespace ispa
