// gemm_tc.cu -- host launchers of the tcgen05 GEMM (statistics and projection).
#define ISPA_DEFINE_GEMM_KERNEL
#include "gemm_tc.cuh"
#include "internal.h"

namespace ispa {

namespace {

ispa_status launch_kernel(const CUtensorMap &ta, const CUtensorMap &tb0, const CUtensorMap &tb1,
                          const CUtensorMap &ta_lo, const CUtensorMap &tb_lo, tcg::Params &P, cudaStream_t s) {
  if (P.n_tiles == 0 || P.K == 0) return ISPA_OK;
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(tcg::gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         tcg::SMEM_BYTES);
    if (e != cudaSuccess) return cuda_status(e, "gemm smem attribute");
    configured_device = dev;
  }
  const int nchunk = P.nchunk > 1 ? P.nchunk : 1;
  tcg::gemm_kernel<<<P.n_tiles * nchunk, tcg::THREADS, tcg::SMEM_BYTES, s>>>(ta, tb0, tb1, ta_lo, tb_lo, P);
  note_launch();
  return cuda_status(cudaGetLastError(), "tcgen05 gemm launch");
}

}  // namespace

ispa_status launch_tc_gemm(const CUtensorMap &ta, const CUtensorMap &tb0, const CUtensorMap &tb1,
                           tcg::Params &P, cudaStream_t s) {
  P.split3 = 0;
  return launch_kernel(ta, tb0, tb1, ta, tb0, P, s);
}

ispa_status launch_tc_gemm_split3(const CUtensorMap &ta, const CUtensorMap &ta_lo, const CUtensorMap &tb,
                                  const CUtensorMap &tb_lo, tcg::Params &P, cudaStream_t s) {
  P.split3 = 1;
  P.n_tiles = P.n_tiles0;  // one sub-problem
  return launch_kernel(ta, tb, tb, ta_lo, tb_lo, P, s);
}

// y[M, N] = A[M, K] B[K, N], A and B bf16 row-major (A K-major, B MN-major).
ispa_status launch_gemm_bf16(int M, int N, int K, const void *A, const void *B, void *Y, ispa_dtype ydt,
                             cudaStream_t s) {
  if (M == 0 || N == 0) return ISPA_OK;
  DevErr err;
  ispa_status st = device_err(&err);
  if (st != ISPA_OK) return st;
  CUtensorMap ta, tb;
  {
    const uint64_t dims[2] = {(uint64_t)K, (uint64_t)M};
    const uint64_t strides[1] = {(uint64_t)K * 2};
    const uint32_t box[2] = {64, 128};
    if ((st = make_tmap(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, A, dims, strides, box,
                        CU_TENSOR_MAP_SWIZZLE_128B)) != ISPA_OK)
      return st;
  }
  bool b_blk = false;
  if ((st = map_mn_blocked(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, B, N, K, N, 64, tcg::BN / 64,
                           CU_TENSOR_MAP_SWIZZLE_128B, &b_blk)) != ISPA_OK)
    return st;
  if (!b_blk) {
    const uint64_t dims[2] = {(uint64_t)N, (uint64_t)K};
    const uint64_t strides[1] = {(uint64_t)N * 2};
    const uint32_t box[2] = {64, 64};
    if ((st = make_tmap(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, B, dims, strides, box,
                        CU_TENSOR_MAP_SWIZZLE_128B)) != ISPA_OK)
      return st;
  }
  tcg::Params P{};
  P.M = M;
  P.K = K;
  P.tiles_m = (M + tcg::BM - 1) / tcg::BM;
  P.kind_tf32 = 0;
  P.a_mn = 0;
  P.b_mn = 1;
  P.idesc = make_idesc(tcg::BM, tcg::BN, 1, 0, 1);
  P.r2 = nullptr;
  P.p[0] = tcg::SubProblem{N, (N + tcg::BN - 1) / tcg::BN, 0,
                           ydt == ISPA_BF16 ? tcg::EPI_STORE_BF16 : tcg::EPI_STORE_F32, Y, N, b_blk ? 1 : 0};
  P.p[1] = P.p[0];
  P.n_tiles0 = P.tiles_m * P.p[0].tiles_n;
  P.n_tiles = P.n_tiles0;
  P.err = err;
  return launch_tc_gemm(ta, tb, tb, P, s);
}

}  // namespace ispa
