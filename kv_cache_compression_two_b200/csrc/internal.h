// internal.h -- host-side declarations shared by the translation units of libispa.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/ispa.h"
#include "common.cuh"

namespace ispa {

// Records a printf-style message as this thread's last error and returns `st`.
ispa_status fail(ispa_status st, const char *fmt, ...);
// ISPA_OK, or ISPA_ERR_CUDA with the CUDA error text.
ispa_status cuda_status(cudaError_t e, const char *what);
// Error word and wait limit of the current device (fetched once per device).
ispa_status device_err(DevErr *out);
// SM count of the current device.
int sm_count();
// The CUDA context current on the calling thread (NULL if none, or if the
// driver entry point is unavailable); keys the caches of device addresses.
void *current_context();

// Encodes a tiled TMA descriptor (driver entry point resolved at run time).
//   dims[0] is the contiguous dimension; strides_bytes has rank-1 entries.
ispa_status make_tmap(CUtensorMap *m, CUtensorMapDataType dt, int rank, const void *base,
                      const uint64_t *dims, const uint64_t *strides_bytes, const uint32_t *box,
                      CUtensorMapSwizzle swizzle);

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Token ranges of the two groups of one attention call (half-open, in rows).
struct GroupRanges {
  int n_loc;            // 0, 1 or 2 local ranges (sink, current), disjoint and ordered
  int loc_begin[2], loc_end[2];
  int hist_begin, hist_end;
  int q_begin;          // first K/V row of the current chunk (queries' own frames)
  int Lq, Lkv;
};

// ---- launchers (each returns ISPA_OK or ISPA_ERR_CUDA) ----
ispa_status launch_lse_merge(int rows, int H, int d, ispa_dtype dt, const void *oa, const float *la,
                             const void *ob, const float *lb, void *oo, float *lo, cudaStream_t s);
// Moves, per instance, the full-layout token rows [b0, b0 + len0) and then
// [b1, b1 + kept_rows - len0) (full_rows rows per instance, row_bytes bytes
// each, a multiple of 16) to the compact layout of kept_rows rows (gather), or
// back from it (scatter; the other full rows are left as they are).
ispa_status launch_kv_remap(int B, long long full_rows, long long kept_rows, long long b0, long long len0,
                            long long b1, long long row_bytes, bool gather, const void *k, const void *v,
                            void *k_out, void *v_out, cudaStream_t s);
// One CTA waiting (bounded by e.limit_ns) on an mbarrier nothing completes.
ispa_status launch_selftest_wait(const DevErr &e, cudaStream_t s);
ispa_status launch_select(int N, const double *eps, int K, unsigned char *is_local, int *idx,
                          cudaStream_t s);
ispa_status launch_absorb_weight(int D, int Dout, const void *W, ispa_dtype wdt, const float *dW,
                                 void *Wn, ispa_dtype odt, cudaStream_t s);
ispa_status launch_attn_simt(const ispa_attn_desc &d, const GroupRanges &g, float scale, const float *q,
                             const float *k, const float *v, void *o_loc, float *l_loc, void *o_hist,
                             float *l_hist, void *o_full, float *l_full, cudaStream_t s);
// workspace: an fp16 copy of V (see attn_tc.cu) plus per-head scales; none
// when V comes prepared (ispa_v16_prepare)
size_t attn_tc_workspace_bytes(int B, int H, int Lkv, int v_layout);
// prepared fp16 V: B * Lkv * H * 128 fp16 values, then the per-head state
size_t v16_bytes(int B, int H, int Lkv);
size_t v16_state_offset(int B, int H, int Lkv);
size_t v16_state_bytes(int B, int H);
// converts rows [row_begin, row_end) of every instance (a prepare from row 0
// clears the state first)
ispa_status launch_v16_prepare(int B, int H, int Lkv, int row_begin, int row_end, const void *v, void *v16,
                               cudaStream_t s);
// fp8 e4m3 attention (attn_f8.cu): the prepared K/V buffer (K8, V8 transposed,
// per-head scales), its prepare, the call's workspace (Q's per-head amax) and
// the launch (kv8 in place of K and V)
size_t kv8_bytes(int B, int H, int Lkv);
size_t attn_f8_workspace_bytes(int B, int H);
ispa_status launch_kv8_prepare(int B, int H, int Lkv, int row_begin, int row_end, const void *k, const void *v,
                               void *kv8, cudaStream_t s);
ispa_status launch_attn_f8(const ispa_attn_desc &d, const GroupRanges &g, float scale, const void *q,
                           const void *kv8, void *o_loc, float *l_loc, void *o_hist, float *l_hist, void *o_full,
                           float *l_full, void *workspace, cudaStream_t s);
ispa_status launch_attn_tc(const ispa_attn_desc &d, const GroupRanges &g, float scale, const void *q,
                           const void *k, const void *v, void *o_loc, float *l_loc, void *o_hist,
                           float *l_hist, void *o_full, float *l_full, void *workspace, cudaStream_t s,
                           float *stats_dA = nullptr);

// stats
size_t stats_workspace_bytes(int T, int D, int Dout, ispa_precision prec);
// rows_ready: the tf32 operands dA and Ar of the rows are already in the workspace
// (written by the attention epilogue); a_loc and a_full are then unused.
ispa_status launch_stats(int T, int D, int Dout, const float *a_loc, const float *a_full, const float *W,
                         float *G, float *C, double *r2, ispa_precision prec, void *ws, cudaStream_t s,
                         bool rows_ready = false);
// Where the attention epilogue puts the operands for launch_stats(rows_ready).
void stats_row_operands(void *ws, int T, int D, int Dout, float **dA, float **Ar);

// ridge
size_t ridge_workspace_bytes(int D, int Dout);
ispa_status launch_ridge(int D, int Dout, const float *G, const float *C, const double *r2, float lambda,
                         int lambda_relative, int refine_steps, float *dW, double *eps, void *ws,
                         cudaStream_t s);
// epsilon of a given dW from statistics (ispa_absorb_error)
size_t absorb_error_workspace_bytes(int D, int Dout);
ispa_status launch_absorb_error(int D, int Dout, const float *G, const float *C, const double *r2, const float *dW,
                                double *eps, void *ws, cudaStream_t s);
// Device address of the static scratch array of ispa_ridge_solve_noalloc on the
// current device, after checking that the workspace of a D x Dout solve fits it.
ispa_status ridge_noalloc_scratch(int D, int Dout, void **out);

// bf16 projection GEMM y[M, N] = A[M, K] * B[K, N] (A, B bf16 row-major) on tcgen05
ispa_status launch_gemm_bf16(int M, int N, int K, const void *A, const void *B, void *Y, ispa_dtype ydt,
                             cudaStream_t s);

// W8A8 projection (quant.cu); fmt is an ispa_q8_format
ispa_status launch_quant_rows(int M, int K, const void *x, int fmt, void *q, float *scale, cudaStream_t s);
ispa_status launch_quant_cols(int K, int N, const void *W, int fmt, void *qT, float *scale, cudaStream_t s);
ispa_status launch_gemm_q8(int M, int N, int K, const void *qa, const float *sa, const void *qT, const float *sw,
                           int fmt, void *y, ispa_dtype ydt, cudaStream_t s);

}  // namespace ispa
