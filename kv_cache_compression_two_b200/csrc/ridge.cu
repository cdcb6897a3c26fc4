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
// One more launch copies L^T from the upper tiles into the lower ones.  Then
// X = L^-1 by recursive 2 x 2 block inversion (batched fp32 GEMMs, one pair
// per recursion depth), and the solve is two triangular GEMMs,
//   dW = X^T (X C),
// fully parallel instead of a chain of block substitutions; the same X serves
// the optional iterative refinement (residual C - (G + lambda I) dW with fp64
// accumulation, dW += X^T (X residual)).  epsilon = r2 - 2<dW, C> + <dW, G dW>
// with fp64 reductions.
//
// The two solve products run on the tensor cores' tf32 pipe: every operand x
// is split into x_hi (the nearest tf32) and x_lo = x - x_hi, and a product is
// taken as A_hi B_hi + A_hi B_lo + A_lo B_hi in three passes of the tcgen05
// GEMM into one fp32 accumulator (the dropped A_lo B_lo and the tf32 rounding
// of the remainders are of order 2^-22 of each term; the accumulator's own
// truncation adds a bias of about 2^-25 of the sum per MMA step).  Their K
// ranges are cut to the triangle of X and split into chunks whose partial
// products are added with atomics.  <dW, G dW> stays on the fp32 CUDA cores:
// epsilon is a small difference of O(r2) terms and needs round-to-nearest
// accumulation.
//
// Sizes are padded to Dp = 64 * ceil(D / 64) with an identity block, which is
// decoupled from the problem and keeps every tile whole.
#include <algorithm>
#include <mutex>
#include <utility>
#include <vector>

#include "gemm_tc.cuh"
#include "internal.h"
#include "simt_gemm.cuh"
#include "simt_gemm_batched.cuh"

namespace ispa {

namespace {

constexpr int NB = 64;

struct Ws {
  float *M;      // [Dp, Dp] lower tiles: G + lambda I, Schur inputs, finally L; upper tiles: L^T
  float *Linv;   // [nb, 64, 64] inverses of the diagonal blocks of L (row-major, lower)
  float *X;      // [Dp, Dp] L^-1 (lower; zero above the diagonal)
  float *T;      // [Dp * Dp / 4] products of the recursive inversion
  float *Y;      // [D, Doutp] L^-1 times the right-hand side
  float *Rres;   // [D, Dout] refinement residual
  float *Bhi;    // [D, Doutp] tf32 parts (nearest tf32, remainder) of a right-hand operand
  float *Blo;
  double *acc;   // [0] <dW, C>  [1] <dW, G dW>  [2] trace(G)  [3] lambda_eff
  int *flag;     // non-zero once a pivot failed
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
int padded(int D) { return (D + NB - 1) / NB * NB; }

int padded4(int n) { return (n + 3) / 4 * 4; }

// Workspace layout; carve() and ridge_workspace_bytes() share it.
size_t carve_bytes(int D, int Dout, Ws *w, void *base) {
  const size_t Dp = (size_t)padded(D);
  char *b = static_cast<char *>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char *q = b ? b + off : nullptr;
    off += align256(bytes);
    return q;
  };
  float *M = reinterpret_cast<float *>(take(Dp * Dp * sizeof(float)));
  float *Linv = reinterpret_cast<float *>(take(Dp * NB * sizeof(float)));
  float *X = reinterpret_cast<float *>(take(Dp * Dp * sizeof(float)));
  float *T = reinterpret_cast<float *>(take(Dp * Dp / 4 * sizeof(float)));
  float *Y = reinterpret_cast<float *>(take((size_t)D * padded4(Dout) * sizeof(float)));
  float *R = reinterpret_cast<float *>(take((size_t)D * Dout * sizeof(float)));
  float *Bhi = reinterpret_cast<float *>(take((size_t)D * padded4(Dout) * sizeof(float)));
  float *Blo = reinterpret_cast<float *>(take((size_t)D * padded4(Dout) * sizeof(float)));
  char *tail = take(256);
  if (w) {
    w->M = M;
    w->Linv = Linv;
    w->X = X;
    w->T = T;
    w->Y = Y;
    w->Rres = R;
    w->Bhi = Bhi;
    w->Blo = Blo;
    w->acc = reinterpret_cast<double *>(tail);
    w->flag = reinterpret_cast<int *>(tail + 64);
  }
  return off;
}

Ws carve(void *base, int D, int Dout) {
  Ws w;
  carve_bytes(D, Dout, &w, base);
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

// (row block, column block) of tile lin of the lower triangle numbered row by
// row: (0,0), (1,0), (1,1), (2,0), ...
__device__ __forceinline__ void lower_tile(int lin, int &I, int &J) {
  int a = (int)((sqrtf(8.f * lin + 1.f) - 1.f) * 0.5f);
  while ((a + 1) * (a + 2) / 2 <= lin) ++a;
  while (a * (a + 1) / 2 > lin) --a;
  I = a;
  J = lin - a * (a + 1) / 2;
}

// M = G + lambda I on the lower tiles (diagonal tiles whole), identity on the
// padding.  One CTA (256 threads) per lower tile: the tile (J, I) of G's upper
// triangle is read row by row into shared memory and written transposed.
__global__ void __launch_bounds__(256) init_kernel(int D, int Dp, const float *__restrict__ G, float lambda,
                                                   int relative, Ws w) {
  const double lam = relative ? (double)lambda * w.acc[2] / D : (double)lambda;
  const float lamf = (float)lam;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    w.acc[0] = 0.0;
    w.acc[1] = 0.0;
    w.acc[3] = (double)lamf;
    *w.flag = 0;
  }
  __shared__ float t[NB][NB + 1];
  int I, J;
  lower_tile(blockIdx.x, I, J);
  for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) {
    const int r = e / NB, c = e % NB, gi = J * NB + r, gj = I * NB + c;
    t[r][c] = (gi < D && gj < D) ? G[(long long)gi * D + gj] : 0.f;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) {
    const int r = e / NB, c = e % NB, i = I * NB + r, j = J * NB + c;
    float x = (I > J || r > c) ? t[c][r] : t[r][c];  // G symmetric from its upper triangle
    if (i == j) x = i < D ? x + lamf : 1.f;
    w.M[(long long)i * Dp + j] = x;
  }
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
  // the swizzled column of a thread is the same for the four rows q0 .. q0 + 3
#pragma unroll 2
  for (int q0 = 0; q0 < NB; q0 += 4) {
    const float *xp = &X[q0][tgrp(ty, q0)], *yp = &Y[q0][tgrp(tx, q0)];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 x = *reinterpret_cast<const float4 *>(xp + i * NB);
      const float4 y = *reinterpret_cast<const float4 *>(yp + i * NB);
      const float xa[4] = {x.x, x.y, x.z, x.w}, yb[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(xa[a], yb[b], acc[a][b]);
    }
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

constexpr int kFactorThreads = 256;
// Steps with at least this many trailing block rows run as two launches (panel,
// update); below it the fused step, whose single launch is shorter on the chain.
constexpr int kTwoLaunchRows = 32;
constexpr int kFactorBcast = 2 * 8 * NB;  // floats of the factor routine's broadcast buffers (two generations)

// Inverse m (lower triangular) of the Cholesky factor of the symmetric 4 x 4
// block d (lower triangle read).  Returns the index of the first non-positive
// pivot, or -1.
__device__ __forceinline__ int chol4_inverse(const float d[4][4], float m[4][4]) {
  const float i0 = rsqrtf(d[0][0]);
  const float l10 = d[1][0] * i0, l20 = d[2][0] * i0, l30 = d[3][0] * i0;
  const float s11 = d[1][1] - l10 * l10;
  const float i1 = rsqrtf(s11);
  const float l21 = (d[2][1] - l20 * l10) * i1, l31 = (d[3][1] - l30 * l10) * i1;
  const float s22 = d[2][2] - l20 * l20 - l21 * l21;
  const float i2 = rsqrtf(s22);
  const float l32 = (d[3][2] - l30 * l20 - l31 * l21) * i2;
  const float s33 = d[3][3] - l30 * l30 - l31 * l31 - l32 * l32;
  const float i3 = rsqrtf(s33);  // NaN after a failed pivot; the result is then discarded
  m[0][0] = i0;
  m[1][1] = i1;
  m[2][2] = i2;
  m[3][3] = i3;
  m[1][0] = -l10 * i0 * i1;
  m[2][1] = -l21 * i1 * i2;
  m[2][0] = -(l20 * i0 + l21 * m[1][0]) * i2;
  m[3][2] = -l32 * i2 * i3;
  m[3][1] = -(l31 * i1 + l32 * m[2][1]) * i3;
  m[3][0] = -(l30 * i0 + l31 * m[1][0] + l32 * m[2][0]) * i3;
  m[0][1] = m[0][2] = m[0][3] = m[1][2] = m[1][3] = m[2][3] = 0.f;
  return !(d[0][0] > 0.f) ? 0 : !(s11 > 0.f) ? 1 : !(s22 > 0.f) ? 2 : !(s33 > 0.f) ? 3 : -1;
}

// Factors the symmetric 64 x 64 matrix S (row-major in shared memory, lower
// triangle and diagonal blocks read, visible to all threads on entry) as
// L L^T and writes L^-1 (row-major, zero above the diagonal) to Linv_out.
// Block forward elimination of [S | I] with Cholesky scaling, four pivots per
// step: with C the four current pivot columns, D their 4 x 4 diagonal block
// and M the inverse of D's Cholesky factor, every row r of the left half below
// the pivots loses l_r l_c^T in column c (l = C M^T), the pivot rows of the
// right half become bn = M times themselves, and every right-half row below
// them loses l_r bn.  Only the lower triangle of the left half below and right
// of the pivots is kept, and the lower triangle of the right half, which ends
// as L^-1.
//
// Ownership: one 4 x 4 block per thread, in registers.  Block column J of the
// left half (block rows J..15) and block row J of the right half left of the
// diagonal (block columns 0..J-1) are 16 blocks, the group of J; warp w holds
// the groups of J = w (lanes 0..15) and J = 15 - w (lanes 16..31), so every
// warp stays busy until its later group is done.  Lane k of group J owns left
// block (J + k, J) for k < 16 - J (k = 0: the diagonal block) and right block
// (J, k - 16 + J) otherwise; the right diagonal block (J, J) is M_J, which
// lane 0 keeps once pivot J is factored.
//
// One barrier per pivot step.  In step P every block still in play applies its
// rank-4 update from the l and bn of pivot P in shared memory.  Right after its
// own update, group P + 1 -- whose blocks are then final for pivot P + 1 --
// factors its diagonal block on lane 0, passes M to the group by shuffles, and
// writes l (left lanes) and bn (right lanes, which keep bn as their final
// value) into the other of two buffers for the next step.  bcast: kFactorBcast
// floats, 16-byte aligned, distinct from S.  kFactorThreads threads.
__device__ __forceinline__ void factor_invert_tile(const float *S, float *bcast, float *__restrict__ Linv_out,
                                                   int pivot_base, int *flag, const DevErr &err) {
  const int t = threadIdx.x, w = t >> 5, lane = t & 31;
  const int J = lane < 16 ? w : 15 - w;  // this lane's group
  const int k = lane & 15;
  const bool left = k < 16 - J;
  const int rb = left ? J + k : J;       // block row of the owned block
  const int cb = left ? J : k - 16 + J;  // block column
  const int last = w > 15 - w ? w : 15 - w;  // the warp has work in steps P < last
  float x[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 v = left ? *reinterpret_cast<const float4 *>(S + (4 * rb + i) * NB + 4 * cb)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
    x[i][0] = v.x;
    x[i][1] = v.y;
    x[i][2] = v.z;
    x[i][3] = v.w;
  }

  // Pivot step Q of group Q; called by the whole warp that holds the group.
  auto pivot = [&](int Q) {
    const bool mine = J == Q;
    if (mine && k == 0) {
      float m[4][4];
      const int bad = chol4_inverse(x, m);
      if (bad >= 0 && atomicExch(flag, 1) == 0) report_error(err, ISPA_ERR_NOT_SPD, pivot_base + 4 * Q + bad + 1);
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) x[a][b] = m[a][b];
    }
    const int src = Q == w ? 0 : 16;
    float mq[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) mq[a][b] = b <= a ? __shfl_sync(0xffffffffu, x[a][b], src) : 0.f;
    float *lb = bcast + (Q & 1) * 8 * NB, *bb = lb + 4 * NB;
    if (!mine) return;
    if (k == 0) {  // the diagonal block of bn is M itself
#pragma unroll
      for (int a = 0; a < 4; ++a)
        *reinterpret_cast<float4 *>(bb + a * NB + 4 * Q) = make_float4(x[a][0], x[a][1], x[a][2], x[a][3]);
    } else if (left) {  // l = C M^T for this block's four rows, component-major
      float l[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          float s = 0.f;
#pragma unroll
          for (int q = 0; q <= jj; ++q) s = fmaf(x[i][q], mq[jj][q], s);
          l[i][jj] = s;
        }
#pragma unroll
      for (int jj = 0; jj < 4; ++jj)
        *reinterpret_cast<float4 *>(lb + jj * NB + 4 * rb) = make_float4(l[0][jj], l[1][jj], l[2][jj], l[3][jj]);
    } else {  // right block (Q, cb): bn = M x, its final value
      float bn[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          float s = 0.f;
#pragma unroll
          for (int q = 0; q <= a; ++q) s = fmaf(mq[a][q], x[q][jj], s);
          bn[a][jj] = s;
        }
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        *reinterpret_cast<float4 *>(bb + a * NB + 4 * cb) = make_float4(bn[a][0], bn[a][1], bn[a][2], bn[a][3]);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) x[a][jj] = bn[a][jj];
      }
    }
  };

  if (w == 0) pivot(0);
  for (int P = 0; P < NB / 4 - 1; ++P) {
    __syncthreads();  // l and bn of pivot P are visible; the buffer written next is no longer read
    if (P >= last) continue;
    if (J > P && (left || cb <= P)) {
      const float *lb = bcast + (P & 1) * 8 * NB;
      const float *vs = (left ? lb : lb + 4 * NB) + 4 * cb;  // l of column block J, or bn at block column cb
      float lr[4][4], v[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const float4 c = *reinterpret_cast<const float4 *>(lb + a * NB + 4 * rb);
        lr[0][a] = c.x;
        lr[1][a] = c.y;
        lr[2][a] = c.z;
        lr[3][a] = c.w;
        const float4 d = *reinterpret_cast<const float4 *>(vs + a * NB);
        v[0][a] = d.x;
        v[1][a] = d.y;
        v[2][a] = d.z;
        v[3][a] = d.w;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          float s = x[i][jj];
#pragma unroll
          for (int a = 0; a < 4; ++a) s = fmaf(-lr[i][a], v[jj][a], s);
          x[i][jj] = s;
        }
    }
    const int q = P + 1;
    if (q == w || q == 15 - w) pivot(q);
  }
  // row J of L^-1: right blocks, M_J on the diagonal, zeros above it
  float *o = Linv_out + (4 * J) * NB;
  if (!left) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<float4 *>(o + i * NB + 4 * cb) = make_float4(x[i][0], x[i][1], x[i][2], x[i][3]);
  } else if (k == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<float4 *>(o + i * NB + 4 * J) = make_float4(x[i][0], x[i][1], x[i][2], x[i][3]);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<float4 *>(o + i * NB + 4 * (J + k)) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// Factor and invert the first diagonal block.  One CTA of kFactorThreads threads.
__global__ void __launch_bounds__(kFactorThreads) chol_first_kernel(int Dp, const float *__restrict__ M, float *Linv,
                                                                     int *flag, DevErr err) {
  __shared__ __align__(16) float S[NB * NB];
  __shared__ __align__(16) float prow[kFactorBcast];
  for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) S[e] = M[(long long)(e / NB) * Dp + e % NB];
  __syncthreads();
  factor_invert_tile(S, prow, Linv, 0, flag, err);
}

// Block step k of the factorisation (see the head of the file).  Grid: one CTA
// per tile of the trailing lower triangle, m (m + 1) / 2 with m = nb - k - 1,
// numbered row by row so that block 0 is the next diagonal tile (k+1, k+1).
// Reads only column-k tiles and Linv_k; writes only trailing tiles, upper
// tiles (k, i) and Linv_{k+1}, so no CTA reads what another CTA writes.
__global__ void __launch_bounds__(kFactorThreads) chol_step_kernel(int Dp, int k, float *M, float *Linv, int *flag,
                                                                    DevErr err) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
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
  float *tile = M + (long long)i * NB * ld + j * NB;

  float aij[4][4];
  load_tile_t(sX, M + (long long)i * NB * ld + k * NB, ld);
  if (!diag) load_tile_t(sY, M + (long long)j * NB * ld + k * NB, ld);
  load_tile_t(sL, Linv + (long long)k * NB * NB, NB);
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
      *reinterpret_cast<float4 *>(S + (4 * ty + a) * NB + 4 * tx) =
          make_float4(aij[a][0], aij[a][1], aij[a][2], aij[a][3]);
    __syncthreads();
    factor_invert_tile(S, &sX[0][0], Linv + (long long)(k + 1) * NB * NB, (k + 1) * NB, flag, err);
  } else {
#pragma unroll
    for (int a = 0; a < 4; ++a)
      *reinterpret_cast<float4 *>(tile + (long long)(4 * ty + a) * ld + 4 * tx) =
          make_float4(aij[a][0], aij[a][1], aij[a][2], aij[a][3]);
  }
}

// Loads the row-major 64 x 64 tile at src into T layout transposed: element
// (row, col) of src becomes element (col, row) of the tile.
__device__ __forceinline__ void load_tile_tt(TileT &T, const float *__restrict__ src, long long ld) {
  const int t = threadIdx.x, c = t & 15;
#pragma unroll
  for (int pass = 0; pass < 4; ++pass) {
    const int q = (t >> 4) + 16 * pass;
    *reinterpret_cast<float4 *>(&T[q][tgrp(c, q)]) = *reinterpret_cast<const float4 *>(src + (long long)q * ld + 4 * c);
  }
}

// Block step k in two launches, for steps with many trailing block rows: the
// fused step above forms each panel tile once per trailing tile that needs it
// (three 64^3 products per CTA, two of them repeated across a block row); here
// chol_panel_kernel forms each L_ik once, and chol_update_kernel applies
// A_ij -= L_ik L_jk^T with one product per CTA.
// Panel: one CTA per block row i > k; writes upper tile (k, i) = L_ik^T.
__global__ void __launch_bounds__(kFactorThreads) chol_panel_kernel(int Dp, int k, float *M, const float *Linv) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ __align__(16) TileT sX;
  __shared__ __align__(16) TileT sL;
  const int i = k + 1 + blockIdx.x;
  const long long ld = Dp;
  load_tile_t(sX, M + (long long)i * NB * ld + k * NB, ld);
  load_tile_t(sL, Linv + (long long)k * NB * NB, NB);
  __syncthreads();
  float p[4][4];
  tile_xyt(sX, sL, p);
  __syncthreads();
  store_acc_t(sX, p);
  __syncthreads();
  const int t = threadIdx.x;
#pragma unroll
  for (int pass = 0; pass < 4; ++pass) {  // row q of the upper tile is column q of L_ik
    const int q = (t >> 4) + 16 * pass, c = t & 15;
    const float4 v = *reinterpret_cast<const float4 *>(&sX[q][tgrp(c, q)]);
    *reinterpret_cast<float4 *>(M + (long long)(k * NB + q) * ld + i * NB + 4 * c) = v;
  }
}

// Update: one CTA per trailing tile (i, j), j <= i, numbered as in
// chol_step_kernel (block 0 is the next diagonal tile, which it then factors and
// inverts for the next step).  Reads upper tiles (k, i), (k, j) and tile (i, j).
__global__ void __launch_bounds__(kFactorThreads) chol_update_kernel(int Dp, int k, float *M, float *Linv, int *flag,
                                                                      DevErr err) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ __align__(16) TileT sX;
  __shared__ __align__(16) TileT sY;
  const int t = threadIdx.x, ty = t >> 4, tx = t & 15;
  const int lin = blockIdx.x;
  int ii = (int)((sqrtf(8.f * lin + 1.f) - 1.f) * 0.5f);
  while ((ii + 1) * (ii + 2) / 2 <= lin) ++ii;
  while (ii * (ii + 1) / 2 > lin) --ii;
  const int i = k + 1 + ii, j = k + 1 + (lin - ii * (ii + 1) / 2);
  const bool diag = i == j;
  const long long ld = Dp;
  float *tile = M + (long long)i * NB * ld + j * NB;
  load_tile_tt(sX, M + (long long)k * NB * ld + i * NB, ld);  // L_ik
  if (!diag) load_tile_tt(sY, M + (long long)k * NB * ld + j * NB, ld);  // L_jk
  float aij[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const float4 v = *reinterpret_cast<const float4 *>(tile + (long long)(4 * ty + a) * ld + 4 * tx);
    aij[a][0] = v.x;
    aij[a][1] = v.y;
    aij[a][2] = v.z;
    aij[a][3] = v.w;
  }
  __syncthreads();
  float upd[4][4];
  tile_xyt(sX, diag ? sX : sY, upd);
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) aij[a][b] -= upd[a][b];
  if (i == k + 1) {
    __syncthreads();  // all reads of sX and sY are done
    float *S = &sY[0][0];
#pragma unroll
    for (int a = 0; a < 4; ++a)
      *reinterpret_cast<float4 *>(S + (4 * ty + a) * NB + 4 * tx) =
          make_float4(aij[a][0], aij[a][1], aij[a][2], aij[a][3]);
    __syncthreads();
    factor_invert_tile(S, &sX[0][0], Linv + (long long)(k + 1) * NB * NB, (k + 1) * NB, flag, err);
  } else {
#pragma unroll
    for (int a = 0; a < 4; ++a)
      *reinterpret_cast<float4 *>(tile + (long long)(4 * ty + a) * ld + 4 * tx) =
          make_float4(aij[a][0], aij[a][1], aij[a][2], aij[a][3]);
  }
}

// Lower tile (i, k) = transpose of upper tile (k, i) for every k < i, after the
// factorisation: the lower triangle then holds L itself (the Schur inputs it
// held are no longer needed), so that both triangular solves read tiles whose
// rows run along the output rows.  One CTA per tile pair, 256 threads.
__global__ void __launch_bounds__(256) upper_to_lower_kernel(int Dp, float *M) {
  __shared__ float s[NB][NB + 1];
  const int lin = blockIdx.x;
  int a = (int)((sqrtf(8.f * lin + 1.f) - 1.f) * 0.5f);
  while ((a + 1) * (a + 2) / 2 <= lin) ++a;
  while (a * (a + 1) / 2 > lin) --a;
  const int i = a + 1, k = lin - a * (a + 1) / 2;  // k <= a < i
  const long long ld = Dp;
  const float *src = M + (long long)k * NB * ld + i * NB;
  float *dst = M + (long long)i * NB * ld + k * NB;
  for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) s[e / NB][e % NB] = src[(e / NB) * ld + e % NB];
  __syncthreads();
  for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) dst[(e / NB) * ld + e % NB] = s[e % NB][e / NB];
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

// out[i][j] = G[min(i,j)][max(i,j)]: the full symmetric matrix from its upper triangle.
__device__ __forceinline__ bool aligned16_dev(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

__device__ __forceinline__ float4 tf32_hi4(float4 x) {
  return make_float4(to_tf32_rn(x.x), to_tf32_rn(x.y), to_tf32_rn(x.z), to_tf32_rn(x.w));
}

// hi = the nearest tf32 of x and lo = x - hi (exact in fp32) for a rows x cols
// block; src and hi may be the same array (then lds == ldd).  Blocks stride
// over rows and threads over the columns of a row, four at a time when every
// leading dimension is a multiple of 4 and every base 16-byte aligned.
__global__ void __launch_bounds__(256) split_tf32_kernel(int rows, int cols, const float *src, long long lds,
                                                         float *hi, float *lo, long long ldd) {
  const bool vec = ((cols | (int)(lds & 3) | (int)(ldd & 3)) & 3) == 0 && aligned16_dev(src) &&
                   aligned16_dev(hi) && aligned16_dev(lo);
  for (int r = blockIdx.x; r < rows; r += gridDim.x) {
    const float *sr = src + (long long)r * lds;
    float *hr = hi + (long long)r * ldd, *lr = lo + (long long)r * ldd;
    if (vec) {
      for (int c = threadIdx.x; c < cols / 4; c += blockDim.x) {
        const float4 x = reinterpret_cast<const float4 *>(sr)[c];
        const float4 h = tf32_hi4(x);
        reinterpret_cast<float4 *>(hr)[c] = h;
        reinterpret_cast<float4 *>(lr)[c] = make_float4(x.x - h.x, x.y - h.y, x.z - h.z, x.w - h.w);
      }
    } else {
      for (int c = threadIdx.x; c < cols; c += blockDim.x) {
        const float x = sr[c], h = to_tf32_rn(x);
        hr[c] = h;
        lr[c] = x - h;
      }
    }
  }
}

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

// acc[1] += <G, P> over a K slice of P = dW dW^T, from the upper triangles of
// both (G's upper triangle as given, weight 2 off the diagonal): equal to
// <dW, G dW> for symmetric G.
struct EpiSymDot {
  const float *G;
  double *acc;
  int ld;
  double part;
  __device__ void begin() { part = 0.0; }
  __device__ void operator()(int m, int n, float a) {
    if (m < n)
      part += 2.0 * (double)G[(long long)m * ld + n] * (double)a;
    else if (m == n)
      part += (double)G[(long long)m * ld + m] * (double)a;
  }
  __device__ void end() {
    const double s = warp_sum_d(part);
    if ((threadIdx.x & 31) == 0) atomicAdd(acc + 1, s);
  }
};

// dst [cols, rows] = src [rows, cols]^T through 32 x 32 shared-memory tiles;
// block (32, 8), grid (ceil(cols / 32), ceil(rows / 32)).
__global__ void transpose_kernel(int rows, int cols, const float *__restrict__ src, long long lds, float *dst,
                                 long long ldd) {
  __shared__ float t[32][33];
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    if (r < rows && c < cols) t[i][threadIdx.x] = src[(long long)r * lds + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int c = c0 + i, r = r0 + threadIdx.x;
    if (r < rows && c < cols) dst[(long long)c * ldd + r] = t[threadIdx.x][i];
  }
}

// out += <a, b> over a rows x cols block with leading dimension ld (fp64
// accumulation); float4 loads when ld is a multiple of 4 and both bases are
// 16-byte aligned.
__global__ void __launch_bounds__(256) dot_kernel(int rows, int cols, long long ld, const float *__restrict__ a,
                                                  const float *__restrict__ b, double *out) {
  const bool vec = ((cols | (int)(ld & 3)) & 3) == 0 && aligned16_dev(a) && aligned16_dev(b);
  double s = 0.0;
  for (int r = blockIdx.x; r < rows; r += gridDim.x) {
    const float *ar = a + (long long)r * ld, *br = b + (long long)r * ld;
    if (vec) {
      for (int c = threadIdx.x; c < cols / 4; c += blockDim.x) {
        const float4 x = reinterpret_cast<const float4 *>(ar)[c], y = reinterpret_cast<const float4 *>(br)[c];
        s += (double)x.x * y.x + (double)x.y * y.y + (double)x.z * y.z + (double)x.w * y.w;
      }
    } else {
      for (int c = threadIdx.x; c < cols; c += blockDim.x) s += (double)ar[c] * (double)br[c];
    }
  }
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

// X = 0 with the inverses of L's diagonal blocks on its diagonal tiles.
// X = the block diagonal of the diagonal-block inverses, zero elsewhere; one
// row per block iteration, four columns per thread (Dp is a multiple of 64).
__global__ void __launch_bounds__(256) x_init_kernel(int Dp, const float *__restrict__ Linv, float *X) {
  for (int r = blockIdx.x; r < Dp; r += gridDim.x) {
    const int rb = r / NB;
    const float4 *lrow = reinterpret_cast<const float4 *>(Linv + (long long)rb * NB * NB + (r % NB) * NB);
    float4 *xrow = reinterpret_cast<float4 *>(X + (long long)r * Dp);
    for (int c = threadIdx.x; c < Dp / 4; c += blockDim.x)
      xrow[c] = (c * 4) / NB == rb ? lrow[c - rb * (NB / 4)] : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// Launches the jobs in batches of kMaxGemmJobs.  With split_k, K is cut into
// chunks so that every SM gets a few CTAs (balancing the triangular K ranges
// and giving the small products of the inversion enough parallelism); the
// outputs must then already hold beta C (zero for beta = 0).
cudaError_t launch_gemm_batch(const GemmJob *jobs, int n, bool split_k, cudaStream_t s) {
  for (int b0 = 0; b0 < n; b0 += kMaxGemmJobs) {
    GemmBatch batch{};
    const int cnt = n - b0 < kMaxGemmJobs ? n - b0 : kMaxGemmJobs;
    int max_m = 0, max_n = 0, max_k = 0, vec = 1;
    long long tiles = 0;
    for (int i = 0; i < cnt; ++i) {
      const GemmJob &j = jobs[b0 + i];
      batch.job[i] = j;
      max_m = max_m > j.M ? max_m : j.M;
      max_n = max_n > j.N ? max_n : j.N;
      max_k = max_k > j.K ? max_k : j.K;
      tiles += (long long)((j.M + 127) / 128) * ((j.N + 127) / 128);
      if ((j.lda | j.ldb) % 4 != 0 || !aligned16(j.A) || !aligned16(j.B)) vec = 0;
    }
    if (max_m == 0 || max_n == 0) continue;
    int nsplit = 1, kchunk = max_k;
    if (split_k && tiles > 0) {
      // chunks of kPipeBK-multiples, about four CTAs per SM in total (the
      // chunks past a tile's triangle are empty, so roughly two do work)
      const long long units = tiles * ((max_k + kPipeBK - 1) / kPipeBK);
      const long long per = units / (4LL * sm_count());
      kchunk = (int)(per > 1 ? per : 1) * kPipeBK;
      nsplit = (max_k + kchunk - 1) / kchunk;
    }
    dim3 grid((max_n + 127) / 128, (max_m + 127) / 128, cnt * nsplit);
    if (vec) {  // 16-byte operands: the cp.async pipeline
      static thread_local int configured_device = -1;
      int dev = 0;
      cudaGetDevice(&dev);
      if (configured_device != dev) {
        cudaError_t e = cudaFuncSetAttribute(simt_gemm_pipe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kPipeSmemBytes);
        if (e != cudaSuccess) return e;
        configured_device = dev;
      }
      simt_gemm_pipe_kernel<<<grid, 256, kPipeSmemBytes, s>>>(batch, nsplit, kchunk);
    } else {
      simt_gemm_batched_kernel<<<grid, 256, 0, s>>>(batch, vec, nsplit, kchunk);
    }
    note_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// X = L^-1 by recursive 2 x 2 block inversion over ranges of diagonal blocks:
//   [L11 0; L21 L22]^-1 = [X11 0; -X22 L21 X11  X22],
// the ranges of one recursion depth combined in one batched launch per
// product, deepest first (the leaves are the diagonal-block inverses).
void split_ranges(int lo, int hi, int depth, std::vector<std::vector<std::pair<int, int>>> &levels) {
  if (hi - lo <= 1) return;
  const int mid = lo + (hi - lo) / 2;
  if ((int)levels.size() <= depth) levels.resize(depth + 1);
  levels[depth].push_back({lo, hi});
  split_ranges(lo, mid, depth + 1, levels);
  split_ranges(mid, hi, depth + 1, levels);
}

cudaError_t invert_factor(int Dp, const Ws &w, cudaStream_t s) {
  const int nb = Dp / NB;
  x_init_kernel<<<sm_count() * 4, 256, 0, s>>>(Dp, w.Linv, w.X);
  note_launch();
  std::vector<std::vector<std::pair<int, int>>> levels;
  split_ranges(0, nb, 0, levels);
  std::vector<GemmJob> first, second;
  for (int d = (int)levels.size() - 1; d >= 0; --d) {
    first.clear();
    second.clear();
    long long t_off = 0;
    for (const auto &r : levels[d]) {
      const int lo = r.first * NB, mid = (r.first + (r.second - r.first) / 2) * NB, hi = r.second * NB;
      const int n1 = mid - lo, n2 = hi - mid;
      float *T = w.T + t_off;  // [n2, n1]
      t_off += (long long)n2 * n1;
      // T = L21 X11   (X11 lower: B[k][n] = 0 for k < n)
      first.push_back(GemmJob{w.M + (long long)mid * Dp + lo, w.X + (long long)lo * Dp + lo, T, Dp, Dp, n1, n2, n1,
                              n1, kTriBLower, 1.f, 0.f});
      // X21 = -X22 T  (X22 lower: A[m][k] = 0 for k > m)
      second.push_back(GemmJob{w.X + (long long)mid * Dp + mid, T, w.X + (long long)mid * Dp + lo, Dp, n1, Dp, n2,
                               n1, n2, kTriALower, -1.f, 0.f});
    }
    // T starts at zero (split-K accumulates into it); X21 is still zero from x_init
    cudaError_t e = cudaMemsetAsync(w.T, 0, (size_t)t_off * sizeof(float), s);
    if (e == cudaSuccess) e = launch_gemm_batch(first.data(), (int)first.size(), true, s);
    if (e == cudaSuccess) e = launch_gemm_batch(second.data(), (int)second.size(), true, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t split_tf32(int rows, int cols, const float *src, long long lds, float *hi, float *lo, long long ldd,
                       cudaStream_t s) {
  split_tf32_kernel<<<sm_count() * 4, 256, 0, s>>>(rows, cols, src, lds, hi, lo, ldd);
  note_launch();
  return cudaGetLastError();
}

// K-tiles (32 elements of K) per CTA of the three-pass products
constexpr int kTc3ChunkKt = 8;

// out += op(A) B on the tf32 pipe: three passes of the tcgen05 GEMM, K chunks
// added with atomics (out must hold its start value).  A is given as its tf32
// parts (a_hi, a_lo), row-major [M, K] with leading dimension lda, or, with
// a_trans, stored [K, M] (op(A) = A^T); B as (b_hi, b_lo), row-major [K, N],
// ldb.  tri cuts each tile's K range to the triangle of op(A) that may be
// non-zero.  Every leading dimension a multiple of 4, every base 16-byte
// aligned.
ispa_status tc3_product(int M, int N, int K, const float *a_hi, const float *a_lo, long long lda, bool a_trans,
                        int tri, const float *b_hi, const float *b_lo, long long ldb, float *out, long long ldo,
                        const DevErr &err, cudaStream_t s) {
  if (M <= 0 || N <= 0 || K <= 0) return ISPA_OK;
  CUtensorMap ta, tal, tb, tbl;
  ispa_status st;
  int a_blk = 0, b_blk = 0;
  if (a_trans) {
    if ((st = map_f32_mn(&ta, a_hi, M, K, lda, 32, tcg::BM / 32, &a_blk)) != ISPA_OK) return st;
    if ((st = map_f32_mn(&tal, a_lo, M, K, lda, 32, tcg::BM / 32, &a_blk)) != ISPA_OK) return st;
  } else {
    if ((st = map2d_f32_ld(&ta, a_hi, K, M, lda, 32, tcg::BM, false)) != ISPA_OK) return st;
    if ((st = map2d_f32_ld(&tal, a_lo, K, M, lda, 32, tcg::BM, false)) != ISPA_OK) return st;
  }
  if ((st = map_f32_mn(&tb, b_hi, N, K, ldb, 32, tcg::BN / 32, &b_blk)) != ISPA_OK) return st;
  if ((st = map_f32_mn(&tbl, b_lo, N, K, ldb, 32, tcg::BN / 32, &b_blk)) != ISPA_OK) return st;
  tcg::Params P{};
  P.M = M;
  P.K = K;
  P.tiles_m = (M + tcg::BM - 1) / tcg::BM;
  P.kind_tf32 = 1;
  P.a_mn = a_trans ? 1 : 0;
  P.b_mn = 1;
  P.a_blk = a_blk;
  P.idesc = make_idesc(tcg::BM, tcg::BN, 2, P.a_mn, 1);
  P.r2 = nullptr;
  P.tri = tri;
  P.chunk_kt = kTc3ChunkKt;
  P.nchunk = ((K + 31) / 32 + kTc3ChunkKt - 1) / kTc3ChunkKt;
  P.p[0] = tcg::SubProblem{N, (N + tcg::BN - 1) / tcg::BN, 0, tcg::EPI_ATOMIC_F32, out, ldo, b_blk};
  P.p[1] = P.p[0];
  P.n_tiles0 = P.tiles_m * P.p[0].tiles_n;
  P.err = err;
  return launch_tc_gemm_split3(ta, tal, tb, tbl, P, s);
}

// out = beta out + A^-1 rhs = beta out + X^T (X rhs), rhs and out [D, Dout]
// (leading dimension Dout, beta 0 or 1), with X in tf32 parts (w.X, w.M).
ispa_status apply_inverse(int D, int Dout, const Ws &w, const float *rhs, float *out, float beta, const DevErr &err,
                          cudaStream_t s) {
  const int Dp = padded(D), ldy = padded4(Dout);
  // the products add their K chunks with atomics: Y starts at zero, out at beta out
  cudaError_t e = split_tf32(D, Dout, rhs, Dout, w.Bhi, w.Blo, ldy, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(w.Y, 0, (size_t)D * ldy * sizeof(float), s);
  if (e == cudaSuccess && beta == 0.f) e = cudaMemsetAsync(out, 0, (size_t)D * Dout * sizeof(float), s);
  if (e != cudaSuccess) return cuda_status(e, "ridge solve set-up");
  // Y = X rhs   (X lower triangular)
  ispa_status st =
      tc3_product(D, Dout, D, w.X, w.M, Dp, false, tcg::TRI_A_LOWER, w.Bhi, w.Blo, ldy, w.Y, ldy, err, s);
  if (st != ISPA_OK) return st;
  e = split_tf32(D, Dout, w.Y, ldy, w.Y, w.Blo, ldy, s);
  if (e != cudaSuccess) return cuda_status(e, "ridge solve split");
  // out += X^T Y   (X^T upper triangular)
  return tc3_product(D, Dout, D, w.X, w.M, Dp, true, tcg::TRI_A_UPPER, w.Y, w.Blo, ldy, out, Dout, err, s);
}

}  // namespace

size_t ridge_workspace_bytes(int D, int Dout) { return carve_bytes(D, Dout, nullptr, nullptr); }

// ---------------------------------------------------------------------------
// epsilon of a given dW on statistics G, C, r2 (ispa_absorb_error): the same
// fp64-accumulated reductions as the solve's epsilon.  Workspace: dW^T and
// two accumulators.
// ---------------------------------------------------------------------------
size_t absorb_error_workspace_bytes(int D, int Dout) { return align256((size_t)Dout * D * sizeof(float)) + 256; }

namespace {
__global__ void eps_finalize_kernel(const double *__restrict__ r2, const double *__restrict__ acc, double *eps) {
  *eps = *r2 - 2.0 * acc[0] + acc[1];
}
}  // namespace

ispa_status launch_absorb_error(int D, int Dout, const float *G, const float *C, const double *r2, const float *dW,
                                double *eps, void *ws, cudaStream_t s) {
  float *dWt = static_cast<float *>(ws);
  double *acc = reinterpret_cast<double *>(static_cast<char *>(ws) + align256((size_t)Dout * D * sizeof(float)));
  cudaError_t e = cudaMemsetAsync(acc, 0, 2 * sizeof(double), s);
  if (e != cudaSuccess) return cuda_status(e, "absorb error set-up");
  const int grid = sm_count() * 4;
  dot_kernel<<<grid, 256, 0, s>>>(D, Dout, Dout, dW, C, acc);
  note_launch();
  if (D % 4 == 0 && Dout % 4 == 0) {
    transpose_kernel<<<dim3((Dout + 31) / 32, (D + 31) / 32), dim3(32, 8), 0, s>>>(D, Dout, dW, Dout, dWt, D);
    note_launch();
    const int tiles = (D + 127) / 128, upper_tiles = tiles * (tiles + 1) / 2;
    const int nsplit = std::max(1, 2 * sm_count() / upper_tiles);
    e = simt_gemm_nn128(D, D, Dout, dW, Dout, dWt, D, EpiSymDot{G, acc, D, 0.0}, s, nsplit, 1);
  } else {
    e = simt_gemm<OP_SYM_UPPER, OP_N, float, 0>(D, Dout, D, Operand{G, nullptr, D}, Operand{dW, nullptr, Dout},
                                                EpiDotG{dW, acc, Dout, 0.0}, s);
  }
  if (e != cudaSuccess) return cuda_status(e, "absorb error G dW");
  eps_finalize_kernel<<<1, 1, 0, s>>>(r2, acc, eps);
  note_launch();
  return cuda_status(cudaGetLastError(), "absorb error launch");
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
// the workspace of the largest size (D a multiple of 64 and Dout of 4, so
// every part is a multiple of 256 bytes): factor copy, inverse, inversion
// products, diagonal-block inverses, four D x Dout buffers, accumulators
constexpr size_t kNoAllocScratchBytes =
    (size_t)ISPA_RIDGE_NOALLOC_MAX_D * ISPA_RIDGE_NOALLOC_MAX_D * 4 * 2 +
    (size_t)ISPA_RIDGE_NOALLOC_MAX_D * ISPA_RIDGE_NOALLOC_MAX_D +
    (size_t)ISPA_RIDGE_NOALLOC_MAX_D * NB * 4 + (size_t)ISPA_RIDGE_NOALLOC_MAX_D * ISPA_RIDGE_NOALLOC_MAX_DOUT * 4 * 4 +
    256;
static __device__ __align__(256) unsigned char g_ridge_scratch[kNoAllocScratchBytes];

ispa_status ridge_noalloc_scratch(int D, int Dout, void **out) {
  const size_t need = carve_bytes(D, Dout, nullptr, nullptr);
  if (need > sizeof(g_ridge_scratch))
    return fail(ISPA_ERR_INVALID_ARG, "ispa_ridge_solve_noalloc: a %d x %d solve needs %zu bytes of scratch, the "
                "static array holds %zu", D, Dout, need, sizeof(g_ridge_scratch));
  static std::mutex mu;
  static void *addr[64] = {};
  static void *ctx_of[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(ISPA_ERR_CUDA, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lock(mu);
  // the address belongs to the context it was looked up in: after a device
  // reset (a new context, the module loaded again) it is looked up afresh
  void *ctx = current_context();
  if (!addr[dev] || !ctx || ctx != ctx_of[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_ridge_scratch);
    if (e != cudaSuccess) return cuda_status(e, "cudaGetSymbolAddress(ridge scratch)");
    addr[dev] = p;
    ctx_of[dev] = current_context();
  }
  *out = addr[dev];
  static_assert(ISPA_RIDGE_NOALLOC_MAX_D % NB == 0 && ISPA_RIDGE_NOALLOC_MAX_DOUT % 64 == 0,
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
  const int Dp = padded(D), nb = Dp / NB;
  const int grid = sm_count() * 4;
  trace_kernel<<<1, 256, 0, s>>>(D, G, w.acc);
  init_kernel<<<nb * (nb + 1) / 2, 256, 0, s>>>(D, Dp, G, lambda, lambda_relative, w);
  chol_first_kernel<<<1, kFactorThreads, 0, s>>>(Dp, w.M, w.Linv, w.flag, err);
  note_launch(3);
  for (int k = 0; k + 1 < nb; ++k) {
    const int m = nb - k - 1;
    // Programmatic dependent launch: a step's grid is set up while the previous
    // step drains (its last CTA is the diagonal factor); each step kernel waits
    // (griddepcontrol.wait) for the previous grid before reading anything.
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kFactorThreads);
    cfg.stream = s;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (m >= kTwoLaunchRows) {  // many trailing tiles: panel once, then one product per tile
      cfg.gridDim = dim3(m);
      cudaError_t le = cudaLaunchKernelEx(&cfg, chol_panel_kernel, Dp, k, w.M, (const float *)w.Linv);
      if (le != cudaSuccess) return cuda_status(le, "ridge factor panel launch");
      cfg.gridDim = dim3(m * (m + 1) / 2);
      le = cudaLaunchKernelEx(&cfg, chol_update_kernel, Dp, k, w.M, w.Linv, w.flag, err);
      if (le != cudaSuccess) return cuda_status(le, "ridge factor update launch");
      note_launch(2);
    } else {
      cfg.gridDim = dim3(m * (m + 1) / 2);
      const cudaError_t le = cudaLaunchKernelEx(&cfg, chol_step_kernel, Dp, k, w.M, w.Linv, w.flag, err);
      if (le != cudaSuccess) return cuda_status(le, "ridge factor step launch");
      note_launch();
    }
  }
  if (nb > 1) {
    upper_to_lower_kernel<<<nb * (nb - 1) / 2, 256, 0, s>>>(Dp, w.M);
    note_launch();
  }
  cudaError_t e = invert_factor(Dp, w, s);
  if (e != cudaSuccess) return cuda_status(e, "ridge inverse");
  // X in tf32 parts for the solve products: hi in place, lo in M (free after the inversion)
  e = split_tf32(Dp, Dp, w.X, Dp, w.X, w.M, Dp, s);
  if (e != cudaSuccess) return cuda_status(e, "ridge inverse split");
  st = apply_inverse(D, Dout, w, C, dW, 0.f, err, s);
  if (st != ISPA_OK) return st;
  const long long nDO = (long long)D * Dout;
  for (int r = 0; r < refine_steps; ++r) {
    e = simt_gemm<OP_SYM_UPPER, OP_N, double, 0>(D, Dout, D, Operand{G, nullptr, D}, Operand{dW, nullptr, Dout},
                                                 EpiResidual{w.Rres, C, dW, w.acc, Dout}, s);
    if (e != cudaSuccess) return cuda_status(e, "ridge residual");
    st = apply_inverse(D, Dout, w, w.Rres, dW, 1.f, err, s);
    if (st != ISPA_OK) return st;
  }
  dot_kernel<<<grid, 256, 0, s>>>(D, Dout, Dout, dW, C, w.acc);
  note_launch();
  // <dW, G dW> on the fp32 CUDA cores: epsilon cancels r2 against 2<dW, C>,
  // so this term needs round-to-nearest accumulation (the tensor cores' fp32
  // accumulation truncates, a bias that grows with K)
  if (D % 4 == 0 && Dout % 4 == 0) {
    // as <G, dW dW^T>: only the upper-triangle tiles of dW dW^T, G read from
    // its upper triangle; dW^T goes to the free right-hand-side buffer, and
    // the K range (Dout) is split so that about two CTAs run per SM
    transpose_kernel<<<dim3((Dout + 31) / 32, (D + 31) / 32), dim3(32, 8), 0, s>>>(D, Dout, dW, Dout, w.Bhi, D);
    note_launch();
    const int tiles = (D + 127) / 128, upper_tiles = tiles * (tiles + 1) / 2;
    const int nsplit = std::max(1, 2 * sm_count() / upper_tiles);
    e = simt_gemm_nn128(D, D, Dout, dW, Dout, w.Bhi, D, EpiSymDot{G, w.acc, D, 0.0}, s, nsplit, 1);
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
