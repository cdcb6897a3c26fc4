// ridge.cu -- closed-form absorption: dW = (G + lambda I)^-1 C and epsilon.
//
// Blocked right-looking Cholesky in fp32 on 64 x 64 tiles, one launch per
// block step k (nb - 1 launches after the first diagonal block):
//   every CTA owns one tile (i, j), k < j <= i, of the trailing lower triangle;
//   it forms the panel tiles it needs itself, L_ik = A_ik Linv_kk^T and
//   L_jk = A_jk Linv_kk^T, and applies A_ij -= L_ik L_jk^T.  The CTA of a
//   diagonal tile (i, i) also stores L_ik^T into the upper tile (k, i), and the
//   CTA of tile (k+1, k+1) -- block 0, dispatched first -- goes on to factor
//   that tile and invert its factor, so the next launch finds Linv_{k+1} ready.
// The lower tiles keep the Schur-complement inputs A_ik; the factor itself is
// kept as U = L^T in the upper tiles plus the inverses of the diagonal blocks,
// which is all the triangular solves read.  Both solves run in ONE launch: the
// right-hand sides are independent, so each CTA takes a panel of 8 columns and
// carries it through the forward (L z = c) and backward (L^T x = z) block
// substitutions in shared memory.  Then optional iterative refinement with
// residuals C - (G + lambda I) X accumulated in fp64, and
// epsilon = r2 - 2<dW, C> + <dW, G dW> with fp64 reductions.
//
// Sizes are padded to Dp = 64 * ceil(D / 64) with an identity block, which is
// decoupled from the problem and keeps every tile whole.
#include <mutex>

#include "internal.h"
#include "simt_gemm.cuh"

namespace ispa {

namespace {

constexpr int NB = 64;
constexpr int kSolveW = 8;   // right-hand-side columns per CTA of the solve
constexpr int kRedLd = 68;   // row stride of the solve's cross-warp partial sums

struct Ws {
  float *M;      // [Dp, Dp] lower tiles: G + lambda I, then Schur inputs; upper tiles: U = L^T
  float *Linv;   // [nb, 64, 64] inverses of the diagonal blocks of L (row-major, lower)
  float *Rres;   // [D, Dout] refinement residual / correction
  double *acc;   // [0] <dW, C>  [1] <dW, G dW>  [2] trace(G)  [3] lambda_eff
  int *flag;     // non-zero once a pivot failed
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
int padded(int D) { return (D + NB - 1) / NB * NB; }

Ws carve(void *base, int D, int Dout) {
  const size_t Dp = (size_t)padded(D);
  char *p = static_cast<char *>(base);
  Ws w;
  w.M = reinterpret_cast<float *>(p);
  p += align256(Dp * Dp * sizeof(float));
  w.Linv = reinterpret_cast<float *>(p);
  p += align256(Dp * NB * sizeof(float));
  w.Rres = reinterpret_cast<float *>(p);
  p += align256((size_t)D * Dout * sizeof(float));
  w.acc = reinterpret_cast<double *>(p);
  p += 64;
  w.flag = reinterpret_cast<int *>(p);
  return w;
}

size_t solve_smem_bytes(int Dp) {
  return sizeof(float) * ((size_t)Dp * kSolveW + 8 * kSolveW * kRedLd + NB * kSolveW + NB * (NB + 1));
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

// M = G + lambda I on the lower tiles (diagonal tiles whole), identity on the
// padding; dW = C as the right-hand side.
__global__ void init_kernel(int D, int Dp, int Dout, const float *__restrict__ G, const float *__restrict__ C,
                            float lambda, int relative, Ws w, float *dW) {
  const double lam = relative ? (double)lambda * w.acc[2] / D : (double)lambda;
  const float lamf = (float)lam;
  const long long nDD = (long long)Dp * Dp, nDO = (long long)D * Dout;
  const long long stride = (long long)gridDim.x * blockDim.x;
  const long long t0 = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (t0 == 0) {
    w.acc[0] = 0.0;
    w.acc[1] = 0.0;
    w.acc[3] = (double)lamf;
    *w.flag = 0;
  }
  for (long long e = t0; e < nDD; e += stride) {
    const int i = (int)(e / Dp), j = (int)(e - (long long)i * Dp);
    if (i / NB < j / NB) continue;  // upper tiles are written by the factorisation
    float x = (i == j) ? 1.f : 0.f;
    if (i < D && j < D) x = G[(long long)min(i, j) * D + max(i, j)] + (i == j ? lamf : 0.f);
    w.M[e] = x;
  }
  for (long long e = t0; e < nDO; e += stride) dW[e] = C[e];
}

// ---------------------------------------------------------------------------
// 64 x 64 tiles in shared memory, "T layout": element (r, q) of a tile X is
// kept in row q at float4 group (r / 4) XOR (q / 4), so that a thread reads
// four consecutive rows of one column as one float4, and the transposing
// stores from row-major global memory spread over the banks.
// ---------------------------------------------------------------------------
using TileT = float[NB][NB];

__device__ __forceinline__ int tgrp(int r4, int q) { return ((r4 ^ (q >> 2)) & 15) << 2; }

// Loads the row-major 64 x 64 tile at src (leading dimension ld) into T layout.
__device__ __forceinline__ void load_tile_t(TileT &T, const float *__restrict__ src, long long ld) {
  const int t = threadIdx.x, c = t & 15;
#pragma unroll
  for (int pass = 0; pass < 4; ++pass) {
    const int r = (t >> 4) + 16 * pass;
    const float4 v = *reinterpret_cast<const float4 *>(src + (long long)r * ld + 4 * c);
    const int col = tgrp(r >> 2, 4 * c) | (r & 3);
    T[4 * c + 0][col] = v.x;
    T[4 * c + 1][col] = v.y;
    T[4 * c + 2][col] = v.z;
    T[4 * c + 3][col] = v.w;
  }
}

// acc[a][b] = sum_q X(4 ty + a, q) Y(4 tx + b, q) for thread (ty, tx) = (t / 16, t % 16).
__device__ __forceinline__ void tile_xyt(const TileT &X, const TileT &Y, float acc[4][4]) {
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
#pragma unroll 8
  for (int q = 0; q < NB; ++q) {
    const float4 x = *reinterpret_cast<const float4 *>(&X[q][tgrp(ty, q)]);
    const float4 y = *reinterpret_cast<const float4 *>(&Y[q][tgrp(tx, q)]);
    const float xa[4] = {x.x, x.y, x.z, x.w}, yb[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(xa[a], yb[b], acc[a][b]);
  }
}

// Stores a product held as acc[a][b] = Z(4 ty + a, 4 tx + b) into T layout.
__device__ __forceinline__ void store_acc_t(TileT &T, const float acc[4][4]) {
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const int q = 4 * tx + b;
    *reinterpret_cast<float4 *>(&T[q][tgrp(ty, q)]) = make_float4(acc[0][b], acc[1][b], acc[2][b], acc[3][b]);
  }
}

// Factors the symmetric 64 x 64 matrix S (row-major in shared memory, only the
// lower triangle read, visible to all threads on entry) as L L^T and writes
// L^-1 (row-major, lower) to Linv_out.  Forward elimination of [S | I] with
// Cholesky scaling turns it into [L^T | L^-1]: at pivot p, row p is divided by
// sqrt(s_pp) and every row r > p loses s_pr / s_pp times the unscaled pivot
// row.  256 threads; thread t owns row r = t / 4 and columns 16 (t % 4) .. +15
// of both halves in registers; the pivot row is published through shared
// memory (prow: 2 x 128 floats, 16-byte aligned, distinct from S; double-
// buffered, so one barrier per pivot).
__device__ void factor_invert_tile(const float *S, float *prow, float *__restrict__ Linv_out, int pivot_base,
                                   int *flag, const DevErr &err) {
  const int t = threadIdx.x, r = t >> 2, c0 = (t & 3) * 16;
  float a[16], b[16];
#pragma unroll
  for (int jj = 0; jj < 16; ++jj) {
    const int c = c0 + jj;
    a[jj] = c <= r ? S[r * NB + c] : S[c * NB + r];
    b[jj] = c == r ? 1.f : 0.f;
  }
  for (int p = 0; p < NB; ++p) {
    float *pr = prow + (p & 1) * 2 * NB;
    if (r == p) {
#pragma unroll
      for (int jj = 0; jj < 16; jj += 4) {
        *reinterpret_cast<float4 *>(pr + c0 + jj) = make_float4(a[jj], a[jj + 1], a[jj + 2], a[jj + 3]);
        *reinterpret_cast<float4 *>(pr + NB + c0 + jj) = make_float4(b[jj], b[jj + 1], b[jj + 2], b[jj + 3]);
      }
    }
    __syncthreads();
    const float d2 = pr[p];
    if (t == 0 && !(d2 > 0.f) && atomicExch(flag, 1) == 0) report_error(err, ISPA_ERR_NOT_SPD, pivot_base + p + 1);
    const float inv = 1.f / sqrtf(d2);  // NaN or inf after a failed pivot; the result is then discarded
    if (r == p) {
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) {
        a[jj] *= inv;
        b[jj] *= inv;
      }
    } else if (r > p) {
      const float g = pr[r] * inv * inv;
#pragma unroll
      for (int jj = 0; jj < 16; jj += 4) {
        const float4 pa = *reinterpret_cast<const float4 *>(pr + c0 + jj);
        const float4 pb = *reinterpret_cast<const float4 *>(pr + NB + c0 + jj);
        a[jj] = fmaf(-g, pa.x, a[jj]);
        a[jj + 1] = fmaf(-g, pa.y, a[jj + 1]);
        a[jj + 2] = fmaf(-g, pa.z, a[jj + 2]);
        a[jj + 3] = fmaf(-g, pa.w, a[jj + 3]);
        b[jj] = fmaf(-g, pb.x, b[jj]);
        b[jj + 1] = fmaf(-g, pb.y, b[jj + 1]);
        b[jj + 2] = fmaf(-g, pb.z, b[jj + 2]);
        b[jj + 3] = fmaf(-g, pb.w, b[jj + 3]);
      }
    }
  }
#pragma unroll
  for (int jj = 0; jj < 16; jj += 4)
    *reinterpret_cast<float4 *>(Linv_out + r * NB + c0 + jj) = make_float4(b[jj], b[jj + 1], b[jj + 2], b[jj + 3]);
}

// Factor and invert the first diagonal block.  One CTA of 256 threads.
__global__ void __launch_bounds__(256) chol_first_kernel(int Dp, const float *__restrict__ M, float *Linv, int *flag,
                                                          DevErr err) {
  __shared__ __align__(16) float S[NB * NB];
  __shared__ __align__(16) float prow[4 * NB];
  for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) S[e] = M[(long long)(e / NB) * Dp + e % NB];
  __syncthreads();
  factor_invert_tile(S, prow, Linv, 0, flag, err);
}

// Block step k of the factorisation (see the head of the file).  Grid: one CTA
// per tile of the trailing lower triangle, m (m + 1) / 2 with m = nb - k - 1,
// numbered row by row so that block 0 is the next diagonal tile (k+1, k+1).
// Reads only column-k tiles and Linv_k; writes only trailing tiles, upper
// tiles (k, i) and Linv_{k+1}, so no CTA reads what another CTA writes.
__global__ void __launch_bounds__(256) chol_step_kernel(int Dp, int k, float *M, float *Linv, int *flag, DevErr err) {
  __shared__ __align__(16) TileT sX;
  __shared__ __align__(16) TileT sY;
  __shared__ __align__(16) TileT sL;
  const int t = threadIdx.x, ty = t >> 4, tx = t & 15;
  const int lin = blockIdx.x;
  int ii = (int)((sqrtf(8.f * lin + 1.f) - 1.f) * 0.5f);
  while ((ii + 1) * (ii + 2) / 2 <= lin) ++ii;
  while (ii * (ii + 1) / 2 > lin) --ii;
  const int i = k + 1 + ii, j = k + 1 + (lin - ii * (ii + 1) / 2);
  const bool diag = i == j;
  const long long ld = Dp;

  load_tile_t(sX, M + (long long)i * NB * ld + k * NB, ld);
  if (!diag) load_tile_t(sY, M + (long long)j * NB * ld + k * NB, ld);
  load_tile_t(sL, Linv + (long long)k * NB * NB, NB);
  float aij[4][4];
  float *tile = M + (long long)i * NB * ld + j * NB;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const float4 v = *reinterpret_cast<const float4 *>(tile + (long long)(4 * ty + a) * ld + 4 * tx);
    aij[a][0] = v.x;
    aij[a][1] = v.y;
    aij[a][2] = v.z;
    aij[a][3] = v.w;
  }
  __syncthreads();

  // panel tiles: L_ik = A_ik Linv_kk^T, L_jk = A_jk Linv_kk^T
  float p1[4][4], p2[4][4];
  tile_xyt(sX, sL, p1);
  if (!diag) tile_xyt(sY, sL, p2);
  __syncthreads();
  store_acc_t(sX, p1);
  if (!diag) store_acc_t(sY, p2);
  __syncthreads();

  if (diag) {
    // upper tile (k, i) = L_ik^T: its row q is column q of L_ik
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
      const int q = (t >> 4) + 16 * pass, c = t & 15;
      const float4 v = *reinterpret_cast<const float4 *>(&sX[q][tgrp(c, q)]);
      *reinterpret_cast<float4 *>(M + (long long)(k * NB + q) * ld + i * NB + 4 * c) = v;
    }
  }

  // trailing update A_ij -= L_ik L_jk^T
  float upd[4][4];
  tile_xyt(sX, diag ? sX : sY, upd);
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) aij[a][b] -= upd[a][b];

  if (i == k + 1) {
    // the next diagonal block: factor and invert it for the next launch
    // (nothing reads the tile itself again, so it is not stored)
    __syncthreads();  // all reads of sX and sY are done
    float *S = &sY[0][0];
#pragma unroll
    for (int a = 0; a < 4; ++a)
      *reinterpret_cast<float4 *>(S + (4 * ty + a) * NB + 4 * tx) = make_float4(aij[a][0], aij[a][1], aij[a][2],
                                                                              aij[a][3]);
    __syncthreads();
    factor_invert_tile(S, &sX[0][0], Linv + (long long)(k + 1) * NB * NB, (k + 1) * NB, flag, err);
  } else {
#pragma unroll
    for (int a = 0; a < 4; ++a)
      *reinterpret_cast<float4 *>(tile + (long long)(4 * ty + a) * ld + 4 * tx) = make_float4(aij[a][0], aij[a][1],
                                                                                            aij[a][2], aij[a][3]);
  }
}

// Both triangular solves for a panel of kSolveW right-hand-side columns, in
// place on X [D, Dout]: forward L z = c (block row b: z_b = Linv_bb (c_b -
// sum over k < 64 b of U[k][64 b + r] z_k)), then backward L^T x = z (x_b =
// Linv_bb^T (z_b - sum over k >= 64 (b + 1) of U[64 b + r][k] x_k)).  The panel
// lives in shared memory for the whole launch.  256 threads (8 warps).
//   forward:  lanes take row pairs of the block (coalesced along a row of U),
//             warps split k; the eight partial sums meet in shared memory.
//   backward: warps take 8 rows each, lanes split k (coalesced along a row of
//             U); a butterfly over the lanes leaves each lane two of the sums.
__global__ void __launch_bounds__(256) chol_solve_kernel(int D, int Dp, int Dout, const float *__restrict__ M,
                                                         const float *__restrict__ Linv, float *X) {
  extern __shared__ __align__(16) float smem[];
  float *z = smem;                                // [Dp][8]
  float *red = z + (size_t)Dp * kSolveW;          // [8 warps][8 columns][kRedLd]
  float *tv = red + 8 * kSolveW * kRedLd;         // [64][8]
  float *sL = tv + NB * kSolveW;                  // [64][65]
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int col0 = blockIdx.x * kSolveW, ncol = min(kSolveW, Dout - col0);
  const int nb = Dp / NB;
  const long long ld = Dp;
  const int r = t >> 2, cc = (t & 3) * 2;  // this thread's two outputs of a block row

  for (int e = t; e < Dp * kSolveW; e += blockDim.x) {
    const int row = e / kSolveW, c = e % kSolveW;
    z[e] = (row < D && c < ncol) ? X[(long long)row * Dout + col0 + c] : 0.f;
  }
  __syncthreads();

  auto stage_linv = [&](int b) {
    const float *src = Linv + (long long)b * NB * NB;
    for (int e = t; e < NB * NB; e += blockDim.x) sL[(e / NB) * (NB + 1) + e % NB] = src[e];
  };

  // ------------------------------------------------------------------ forward
  for (int b = 0; b < nb; ++b) {
    const int rb = b * NB;
    float acc[2][kSolveW];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int c = 0; c < kSolveW; ++c) acc[i][c] = 0.f;
    const float *ucol = M + rb + 2 * lane;
#pragma unroll 4
    for (int k = warp; k < rb; k += 8) {
      const float2 u = *reinterpret_cast<const float2 *>(ucol + (long long)k * ld);
      const float4 z0 = *reinterpret_cast<const float4 *>(z + k * kSolveW);
      const float4 z1 = *reinterpret_cast<const float4 *>(z + k * kSolveW + 4);
      const float zk[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
#pragma unroll
      for (int c = 0; c < kSolveW; ++c) {
        acc[0][c] = fmaf(u.x, zk[c], acc[0][c]);
        acc[1][c] = fmaf(u.y, zk[c], acc[1][c]);
      }
    }
#pragma unroll
    for (int c = 0; c < kSolveW; ++c)
      *reinterpret_cast<float2 *>(red + (warp * kSolveW + c) * kRedLd + 2 * lane) = make_float2(acc[0][c], acc[1][c]);
    stage_linv(b);
    __syncthreads();
    {
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        s0 += red[(w * kSolveW + cc) * kRedLd + r];
        s1 += red[(w * kSolveW + cc + 1) * kRedLd + r];
      }
      const float2 zc = *reinterpret_cast<const float2 *>(z + (rb + r) * kSolveW + cc);
      *reinterpret_cast<float2 *>(tv + r * kSolveW + cc) = make_float2(zc.x - s0, zc.y - s1);
    }
    __syncthreads();
    {
      float o0 = 0.f, o1 = 0.f;
#pragma unroll 8
      for (int q = 0; q < NB; ++q) {
        const float l = sL[r * (NB + 1) + q];
        const float2 v = *reinterpret_cast<const float2 *>(tv + q * kSolveW + cc);
        o0 = fmaf(l, v.x, o0);
        o1 = fmaf(l, v.y, o1);
      }
      *reinterpret_cast<float2 *>(z + (rb + r) * kSolveW + cc) = make_float2(o0, o1);
    }
    __syncthreads();
  }

  // ----------------------------------------------------------------- backward
  for (int b = nb - 1; b >= 0; --b) {
    const int rb = b * NB;
    float v[64];  // v[i * 8 + c]: row rb + 8 warp + i, column c
#pragma unroll
    for (int e = 0; e < 64; ++e) v[e] = 0.f;
    const float *urow = M + (long long)(rb + 8 * warp) * ld;
#pragma unroll 2
    for (int k = rb + NB + lane; k < Dp; k += 32) {
      const float4 z0 = *reinterpret_cast<const float4 *>(z + k * kSolveW);
      const float4 z1 = *reinterpret_cast<const float4 *>(z + k * kSolveW + 4);
      const float zk[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float u = urow[(long long)i * ld + k];
#pragma unroll
        for (int c = 0; c < kSolveW; ++c) v[i * 8 + c] = fmaf(u, zk[c], v[i * 8 + c]);
      }
    }
    // reduce-scatter over the lanes: afterwards lane l holds the sums of
    // entries 2 l and 2 l + 1, i.e. row 8 warp + l / 4, columns 2 (l % 4) + {0, 1}
#pragma unroll
    for (int lvl = 0; lvl < 5; ++lvl) {
      const int half = 32 >> lvl, off = 16 >> lvl;
      const bool upper = (lane & off) != 0;
#pragma unroll
      for (int m = 0; m < half; ++m) {
        const float keep = upper ? v[half + m] : v[m];
        const float send = upper ? v[m] : v[half + m];
        v[m] = keep + __shfl_xor_sync(0xffffffffu, send, off);
      }
    }
    stage_linv(b);
    {
      const float2 zc = *reinterpret_cast<const float2 *>(z + (rb + r) * kSolveW + cc);
      *reinterpret_cast<float2 *>(tv + r * kSolveW + cc) = make_float2(zc.x - v[0], zc.y - v[1]);
    }
    __syncthreads();
    {
      float o0 = 0.f, o1 = 0.f;
#pragma unroll 8
      for (int q = 0; q < NB; ++q) {
        const float l = sL[q * (NB + 1) + r];
        const float2 w2 = *reinterpret_cast<const float2 *>(tv + q * kSolveW + cc);
        o0 = fmaf(l, w2.x, o0);
        o1 = fmaf(l, w2.y, o1);
      }
      *reinterpret_cast<float2 *>(z + (rb + r) * kSolveW + cc) = make_float2(o0, o1);
    }
    __syncthreads();
  }

  for (int e = t; e < D * kSolveW; e += blockDim.x) {
    const int row = e / kSolveW, c = e % kSolveW;
    if (c < ncol) X[(long long)row * Dout + col0 + c] = z[e];
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

// Solves (G + lambda I) X = Y in place on Y [D, Dout] with the factorisation in w.
cudaError_t cholesky_solve(int D, int Dout, const Ws &w, float *Y, cudaStream_t s) {
  const int Dp = padded(D);
  const size_t smem = solve_smem_bytes(Dp);
  cudaError_t e = cudaFuncSetAttribute(chol_solve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  chol_solve_kernel<<<(Dout + kSolveW - 1) / kSolveW, 256, smem, s>>>(D, Dp, Dout, w.M, w.Linv, Y);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

size_t ridge_workspace_bytes(int D, int Dout) {
  const size_t Dp = (size_t)padded(D);
  return align256(Dp * Dp * sizeof(float)) + align256(Dp * NB * sizeof(float)) +
         align256((size_t)D * Dout * sizeof(float)) + 256;
}

int ridge_max_dim() {
  // the solve keeps a Dp x 8 panel in shared memory
  int dev = 0, optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return 0;
  const size_t fixed = solve_smem_bytes(0);
  if ((size_t)optin <= fixed) return 0;
  return (int)(((size_t)optin - fixed) / (sizeof(float) * kSolveW)) / NB * NB;
}

// ---------------------------------------------------------------------------
// Allocation-free variant (ispa_ridge_solve_noalloc).  Its scratch -- the
// working copy of the factorisation, the refinement residual and a few
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
  static_assert(ISPA_RIDGE_NOALLOC_MAX_D % NB == 0, "the largest workspace must fit the scratch exactly");
  return ISPA_OK;
}

ispa_status launch_ridge(int D, int Dout, const float *G, const float *C, const double *r2, float lambda,
                         int lambda_relative, int refine_steps, float *dW, double *eps, void *ws_base,
                         cudaStream_t s) {
  DevErr err;
  ispa_status st = device_err(&err);
  if (st != ISPA_OK) return st;
  Ws w = carve(ws_base, D, Dout);
  const int Dp = padded(D), nb = Dp / NB;
  const int grid = sm_count() * 4;
  trace_kernel<<<1, 256, 0, s>>>(D, G, w.acc);
  init_kernel<<<grid, 256, 0, s>>>(D, Dp, Dout, G, C, lambda, lambda_relative, w, dW);
  chol_first_kernel<<<1, 256, 0, s>>>(Dp, w.M, w.Linv, w.flag, err);
  note_launch(3);
  for (int k = 0; k + 1 < nb; ++k) {
    const int m = nb - k - 1;
    chol_step_kernel<<<m * (m + 1) / 2, 256, 0, s>>>(Dp, k, w.M, w.Linv, w.flag, err);
    note_launch();
  }
  cudaError_t e = cholesky_solve(D, Dout, w, dW, s);
  if (e != cudaSuccess) return cuda_status(e, "ridge solve");
  const long long nDO = (long long)D * Dout;
  for (int r = 0; r < refine_steps; ++r) {
    e = simt_gemm<OP_SYM_UPPER, OP_N, double, 0>(D, Dout, D, Operand{G, nullptr, D}, Operand{dW, nullptr, Dout},
                                                 EpiResidual{w.Rres, C, dW, w.acc, Dout}, s);
    if (e != cudaSuccess) return cuda_status(e, "ridge residual");
    e = cholesky_solve(D, Dout, w, w.Rres, s);
    if (e != cudaSuccess) return cuda_status(e, "ridge refinement solve");
    add_kernel<<<grid, 256, 0, s>>>(nDO, dW, w.Rres);
    note_launch();
  }
  dot_kernel<<<grid, 256, 0, s>>>(nDO, dW, C, w.acc);
  note_launch();
  if (D % 4 == 0 && Dout % 4 == 0) {
    // the factorisation is no longer needed: expand G to the full symmetric
    // matrix there so that the G dW product reads both operands row-major with
    // 16-byte loads
    symmetrize_kernel<<<grid, 256, 0, s>>>(D, G, w.M);
    note_launch();
    e = simt_gemm_nn128(D, Dout, D, w.M, D, dW, Dout, EpiDotG{dW, w.acc, Dout, 0.0}, s);
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
