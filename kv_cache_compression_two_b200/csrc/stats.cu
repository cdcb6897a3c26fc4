// stats.cu -- warmup accumulation of the absorption statistics.
//
//   R = (A_full - A_loc) W,  G += A_loc^T A_loc (upper triangle),  C += A_loc^T R,  r2 += ||R||^2
//
// ISPA_PREC_TF32 (tcgen05): a streaming pass rounds dA = A_full - A_loc, A_loc
// and W to the nearest tf32 (round-to-nearest keeps the products unbiased;
// the tensor core would otherwise truncate), then
//   launch 1: R = dA W                 (A K-major, B MN-major), epilogue stores
//             tf32(R) and adds ||R||^2 in fp64;
//   launch 2: [G | C] += A_loc^T [A_loc | R]   (both operands MN-major, i.e.
//             A_loc read row-major with no transpose pass; only the tiles of
//             G on or above the diagonal are computed).
// ISPA_PREC_F32: the same three products on the fp32 CUDA cores.
#include "gemm_tc.cuh"
#include "internal.h"
#include "simt_gemm.cuh"

namespace ispa {

namespace {

size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

__global__ void __launch_bounds__(256) prep_tf32_kernel(long long n4_rows, long long n4_w,
                                                        const float4 *__restrict__ a_loc,
                                                        const float4 *__restrict__ a_full,
                                                        const float4 *__restrict__ W, float4 *dA, float4 *Ar,
                                                        float4 *Wr) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4_rows; i += stride) {
    const float4 l = __ldcs(a_loc + i), f = __ldcs(a_full + i);
    dA[i] = make_float4(to_tf32_rn(f.x - l.x), to_tf32_rn(f.y - l.y), to_tf32_rn(f.z - l.z), to_tf32_rn(f.w - l.w));
    Ar[i] = make_float4(to_tf32_rn(l.x), to_tf32_rn(l.y), to_tf32_rn(l.z), to_tf32_rn(l.w));
  }
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4_w; i += stride) {
    const float4 w = __ldg(W + i);
    Wr[i] = make_float4(to_tf32_rn(w.x), to_tf32_rn(w.y), to_tf32_rn(w.z), to_tf32_rn(w.w));
  }
}

// R = dA W in the fp32 path: store R, accumulate ||R||^2.
struct EpiStoreSq {
  float *out;
  int ld;
  double *r2;
  double part;
  __device__ void begin() { part = 0.0; }
  __device__ void operator()(int m, int n, float a) {
    out[(long long)m * ld + n] = a;
    part += (double)a * a;
  }
  __device__ void end() {
    const double s = warp_sum_d(part);
    if ((threadIdx.x & 31) == 0) atomicAdd(r2, s);
  }
};

struct TF32Ws {
  float *dA, *Ar, *Wr, *R;
};

TF32Ws carve_tf32(void *ws, int T, int D, int Dout) {
  char *p = static_cast<char *>(ws);
  TF32Ws w;
  w.dA = reinterpret_cast<float *>(p);
  p += a256((size_t)T * D * 4);
  w.Ar = reinterpret_cast<float *>(p);
  p += a256((size_t)T * D * 4);
  w.Wr = reinterpret_cast<float *>(p);
  p += a256((size_t)D * Dout * 4);
  w.R = reinterpret_cast<float *>(p);
  return w;
}

}  // namespace

size_t stats_workspace_bytes(int T, int D, int Dout, ispa_precision prec) {
  if (prec == ISPA_PREC_F32) return a256((size_t)T * Dout * 4);
  return 2 * a256((size_t)T * D * 4) + a256((size_t)D * Dout * 4) + a256((size_t)T * Dout * 4);
}

void stats_row_operands(void *ws, int T, int D, int Dout, float **dA, float **Ar) {
  TF32Ws w = carve_tf32(ws, T, D, Dout);
  *dA = w.dA;
  *Ar = w.Ar;
}

ispa_status launch_stats(int T, int D, int Dout, const float *a_loc, const float *a_full, const float *W,
                         float *G, float *C, double *r2, ispa_precision prec, void *ws, cudaStream_t s,
                         bool rows_ready) {
  if (T == 0) return ISPA_OK;
  if (prec == ISPA_PREC_F32) {
    float *R = static_cast<float *>(ws);
    cudaError_t e = simt_gemm<OP_N, OP_N, float, 0>(T, Dout, D, Operand{a_full, a_loc, D}, Operand{W, nullptr, Dout},
                                                    EpiStoreSq{R, Dout, r2, 0.0}, s);
    if (e == cudaSuccess)
      e = simt_gemm<OP_T, OP_N, float, 2>(D, D, T, Operand{a_loc, nullptr, D}, Operand{a_loc, nullptr, D},
                                          EpiAxpby{G, D, 1.f, 1.f, 2}, s);
    if (e == cudaSuccess)
      e = simt_gemm<OP_T, OP_N, float, 0>(D, Dout, T, Operand{a_loc, nullptr, D}, Operand{R, nullptr, Dout},
                                          EpiAxpby{C, Dout, 1.f, 1.f, 0}, s);
    return cuda_status(e, "stats (fp32) launch");
  }

  DevErr err;
  ispa_status st = device_err(&err);
  if (st != ISPA_OK) return st;
  TF32Ws w = carve_tf32(ws, T, D, Dout);
  const long long n4_rows = rows_ready ? 0 : (long long)T * D / 4, n4_w = (long long)D * Dout / 4;
  prep_tf32_kernel<<<sm_count() * 8, 256, 0, s>>>(n4_rows, n4_w, (const float4 *)a_loc, (const float4 *)a_full,
                                                  (const float4 *)W, (float4 *)w.dA, (float4 *)w.Ar, (float4 *)w.Wr);
  note_launch();
  st = cuda_status(cudaGetLastError(), "stats prep launch");
  if (st != ISPA_OK) return st;

  // launch 1: R = dA W
  {
    CUtensorMap ta, tb;
    int b_blk = 0;
    if ((st = map2d_f32(&ta, w.dA, D, T, 32, 128, false)) != ISPA_OK) return st;
    if ((st = map_f32_mn(&tb, w.Wr, Dout, D, Dout, 32, tcg::BN / 32, &b_blk)) != ISPA_OK) return st;
    tcg::Params P{};
    P.M = T;
    P.K = D;
    P.tiles_m = (T + tcg::BM - 1) / tcg::BM;
    P.kind_tf32 = 1;
    P.a_mn = 0;
    P.b_mn = 1;
    P.idesc = make_idesc(tcg::BM, tcg::BN, 2, 0, 1);
    P.r2 = r2;
    P.p[0] = tcg::SubProblem{Dout, (Dout + tcg::BN - 1) / tcg::BN, 0, tcg::EPI_STORE_TF32_SQ, w.R, Dout, b_blk};
    P.n_tiles0 = P.tiles_m * P.p[0].tiles_n;
    P.n_tiles = P.n_tiles0;
    P.p[1] = P.p[0];
    P.err = err;
    if ((st = launch_tc_gemm(ta, tb, tb, P, s)) != ISPA_OK) return st;
  }
  // launch 2: G (upper) += Ar^T Ar, C += Ar^T R
  {
    // Ar is A (128-wide tiles) and the B of G (256-wide tiles): one map each
    CUtensorMap ta, tg, tr;
    int a_blk = 0, g_blk = 0, r_blk = 0;
    if ((st = map_f32_mn(&ta, w.Ar, D, T, D, 32, tcg::BM / 32, &a_blk)) != ISPA_OK) return st;
    if ((st = map_f32_mn(&tg, w.Ar, D, T, D, 32, tcg::BN / 32, &g_blk)) != ISPA_OK) return st;
    if ((st = map_f32_mn(&tr, w.R, Dout, T, Dout, 32, tcg::BN / 32, &r_blk)) != ISPA_OK) return st;
    tcg::Params P{};
    P.M = D;
    P.K = T;
    P.tiles_m = (D + tcg::BM - 1) / tcg::BM;
    P.kind_tf32 = 1;
    P.a_mn = 1;
    P.b_mn = 1;
    P.a_blk = a_blk;
    P.idesc = make_idesc(tcg::BM, tcg::BN, 2, 1, 1);
    P.r2 = nullptr;
    P.p[0] = tcg::SubProblem{D, (D + tcg::BN - 1) / tcg::BN, 1, tcg::EPI_ACCUM_F32, G, D, g_blk};
    P.p[1] = tcg::SubProblem{Dout, (Dout + tcg::BN - 1) / tcg::BN, 0, tcg::EPI_ACCUM_F32, C, Dout, r_blk};
    P.n_tiles0 = tcg::upper_tile_count(P.tiles_m, P.p[0].tiles_n);
    P.n_tiles = P.n_tiles0 + P.tiles_m * P.p[1].tiles_n;
    P.err = err;
    if ((st = launch_tc_gemm(ta, tg, tr, P, s)) != ISPA_OK) return st;
  }
  return ISPA_OK;
}

}  // namespace ispa
