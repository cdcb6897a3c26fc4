// quant.cu -- 8-bit (W8A8) post-switch projection: per-row / per-column
// quantisation and the 8-bit tcgen05 product.
//
// The paper combines ISPA with post-training W8A8 quantisation and reports the
// combined speed-up ([EN-notes] "Key Findings", Figure 7; [DE-summary] §4
// "Beschleunigung").  The pages do not fix the scheme; this file takes the
// plain symmetric one: every activation row (token) and every weight column
// (output channel) gets one scale s = amax / QMAX, values are x / s rounded to
// the 8-bit format, and y[m, n] = (sum_k qa[m, k] qw[k, n]) * sa[m] * sw[n].
//   e4m3:  QMAX = 448, round to nearest even with saturation (cvt.rn.satfinite)
//   int8:  QMAX = 127, round half to even, clamped to [-127, 127]; the int8
//          product accumulates exactly in int32 on kind::i8.
// The quantiser multiplies by inv = QMAX / amax (fp32, rounded) rather than
// dividing by s; a row or column of zeros gets s = 0, inv = 0 and q = 0.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "gemm_tc.cuh"
#include "internal.h"

namespace ispa {
namespace {

constexpr float kQmaxE4m3 = 448.f, kQmaxS8 = 127.f;

__device__ __forceinline__ uint32_t quant1(float x, int fmt) {
  if (fmt == ISPA_Q8_E4M3) return (uint32_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
  const int q = max(-127, min(127, __float2int_rn(x)));
  return (uint32_t)(uint8_t)(int8_t)q;
}

__device__ __forceinline__ void unpack_bf16x8(const uint4 &u, float (&x)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// One warp per row of x [M, K] (bf16, K % 16 == 0): amax, then the quantised
// row q [M, K] (one byte per value) and its scale.
__global__ void __launch_bounds__(256) quant_rows_kernel(int M, int K, const __nv_bfloat16 *__restrict__ x,
                                                         int fmt, uint8_t *__restrict__ q,
                                                         float *__restrict__ scale) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= M) return;
  const uint4 *xr = reinterpret_cast<const uint4 *>(x + (long long)row * K);
  const int nv = K / 8;
  float amax = 0.f;
  for (int v = lane; v < nv; v += 32) {
    float f[8];
    unpack_bf16x8(__ldg(xr + v), f);
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float qmax = fmt == ISPA_Q8_E4M3 ? kQmaxE4m3 : kQmaxS8;
  const float inv = amax > 0.f ? __fdiv_rn(qmax, amax) : 0.f;
  uint2 *qr = reinterpret_cast<uint2 *>(q + (long long)row * K);
  for (int v = lane; v < nv; v += 32) {
    float f[8];
    unpack_bf16x8(__ldg(xr + v), f);
    uint32_t b[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) b[i] = quant1(__fmul_rn(f[i], inv), fmt);
    qr[v] = make_uint2(b[0] | b[1] << 8 | b[2] << 16 | b[3] << 24, b[4] | b[5] << 8 | b[6] << 16 | b[7] << 24);
  }
  if (lane == 0) scale[row] = __fdiv_rn(amax, qmax);
}

// W [K, N] (bf16, row-major) -> qT [N, K] (one byte per value, K-major) with
// one scale per column n.  A CTA of 32 x 8 threads owns 32 columns: pass 1
// takes their amax over all K rows, pass 2 quantises 32 x 32 blocks and writes
// them transposed through shared memory.
__global__ void __launch_bounds__(256) quant_cols_kernel(int K, int N, const __nv_bfloat16 *__restrict__ W,
                                                         int fmt, uint8_t *__restrict__ qT,
                                                         float *__restrict__ scale) {
  __shared__ float red[8][32];
  __shared__ uint8_t tile[32][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int n0 = blockIdx.x * 32, n = n0 + tx;
  float amax = 0.f;
  if (n < N)
    for (int k = ty; k < K; k += 8) amax = fmaxf(amax, fabsf(__bfloat162float(W[(long long)k * N + n])));
  red[ty][tx] = amax;
  __syncthreads();
  if (ty == 0) {
    for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i][tx]);
    red[0][tx] = amax;
  }
  __syncthreads();
  const float qmax = fmt == ISPA_Q8_E4M3 ? kQmaxE4m3 : kQmaxS8;
  const float cmax = red[0][tx];
  const float inv = cmax > 0.f ? __fdiv_rn(qmax, cmax) : 0.f;
  if (ty == 0 && n < N) scale[n] = __fdiv_rn(cmax, qmax);
  // writer mapping: thread t stores bytes [4 (t % 8), +4) of row t / 8 of the transposed block
  const int wn = threadIdx.x >> 3, wk = (threadIdx.x & 7) * 4;
  for (int k0 = 0; k0 < K; k0 += 32) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int kk = ty + 8 * i, k = k0 + kk;
      tile[tx][kk] = (n < N && k < K) ? (uint8_t)quant1(__fmul_rn(__bfloat162float(W[(long long)k * N + n]), inv), fmt)
                                      : (uint8_t)0;
    }
    __syncthreads();
    if (n0 + wn < N && k0 + wk < K) {
      const uint32_t v = (uint32_t)tile[wn][wk] | (uint32_t)tile[wn][wk + 1] << 8 |
                         (uint32_t)tile[wn][wk + 2] << 16 | (uint32_t)tile[wn][wk + 3] << 24;
      *reinterpret_cast<uint32_t *>(qT + (long long)(n0 + wn) * K + k0 + wk) = v;
    }
    __syncthreads();
  }
}

}  // namespace

ispa_status launch_quant_rows(int M, int K, const void *x, int fmt, void *q, float *scale, cudaStream_t s) {
  if (M == 0) return ISPA_OK;
  quant_rows_kernel<<<(M + 7) / 8, 256, 0, s>>>(M, K, static_cast<const __nv_bfloat16 *>(x), fmt,
                                                 static_cast<uint8_t *>(q), scale);
  note_launch();
  return cuda_status(cudaGetLastError(), "quant_rows launch");
}

ispa_status launch_quant_cols(int K, int N, const void *W, int fmt, void *qT, float *scale, cudaStream_t s) {
  if (N == 0) return ISPA_OK;
  quant_cols_kernel<<<(N + 31) / 32, 256, 0, s>>>(K, N, static_cast<const __nv_bfloat16 *>(W), fmt,
                                                   static_cast<uint8_t *>(qT), scale);
  note_launch();
  return cuda_status(cudaGetLastError(), "quant_cols launch");
}

// y[M, N] = (qa[M, K] qw[K, N]) * sa[m] * sw[n], both operands 8-bit K-major
// (qa row-major [M, K], qw given as its transpose qT [N, K]).
ispa_status launch_gemm_q8(int M, int N, int K, const void *qa, const float *sa, const void *qT, const float *sw,
                           int fmt, void *y, ispa_dtype ydt, cudaStream_t s) {
  if (M == 0 || N == 0) return ISPA_OK;
  DevErr err;
  ispa_status st = device_err(&err);
  if (st != ISPA_OK) return st;
  // A: 128-row boxes; B: one 256-row box per stage (the copy engine's time is
  // mostly per box, so a stage in fewer boxes arrives sooner)
  CUtensorMap ta, tb;
  const uint64_t strides[1] = {(uint64_t)K};
  {
    const uint64_t dims[2] = {(uint64_t)K, (uint64_t)M};
    const uint32_t box[2] = {128, (uint32_t)tcg::BM};
    if ((st = make_tmap(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, qa, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) !=
        ISPA_OK)
      return st;
  }
  {
    const uint64_t dims[2] = {(uint64_t)K, (uint64_t)N};
    const uint32_t box[2] = {128, (uint32_t)tcg::BN};
    if ((st = make_tmap(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, qT, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) !=
        ISPA_OK)
      return st;
  }
  tcg::Params P{};
  P.M = M;
  P.K = K;
  P.tiles_m = (M + tcg::BM - 1) / tcg::BM;
  P.kind_tf32 = 0;
  P.kind_f8 = fmt == ISPA_Q8_E4M3 ? 1 : 2;
  P.a_mn = 0;
  P.b_mn = 0;
  P.idesc = fmt == ISPA_Q8_E4M3 ? make_idesc(tcg::BM, tcg::BN, 0, 0, 0) : make_idesc_s8(tcg::BM, tcg::BN);
  P.row_scale = sa;
  P.col_scale = sw;
  P.out_bf16 = ydt == ISPA_BF16;
  P.p[0] = tcg::SubProblem{N, (N + tcg::BN - 1) / tcg::BN, 0, tcg::EPI_SCALED, y, N, 1};
  P.p[1] = P.p[0];
  P.n_tiles0 = P.tiles_m * P.p[0].tiles_n;
  P.n_tiles = P.n_tiles0;
  P.err = err;
  return launch_tc_gemm(ta, tb, tb, P, s);
}

}  // namespace ispa
