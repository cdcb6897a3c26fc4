// elementwise.cu -- HBM-bound kernels: LSE merge, weight correction, layer selection.
#include "internal.h"

namespace ispa {

// ---------------------------------------------------------------------------
// LSE merge of two disjoint attention groups.
//   L = log(e^La + e^Lb),  O = e^(La-L) Oa + e^(Lb-L) Ob
// One thread moves one 16-byte vector of O (4 fp32 or 8 bf16); the head's two
// LSE values are broadcast loads that hit L1.  Grid-stride over all vectors.
// ---------------------------------------------------------------------------
struct MergeW {
  float wa, wb, L;
};

__device__ __forceinline__ MergeW merge_weights(float la, float lb) {
  MergeW r;
  const float m = fmaxf(la, lb);
  if (m == -INFINITY) {
    r.wa = 0.f;
    r.wb = 0.f;
    r.L = -INFINITY;
    return r;
  }
  const float ea = expf(la - m), eb = expf(lb - m);
  const float s = ea + eb;
  r.L = m + logf(s);
  const float inv = 1.f / s;
  r.wa = ea * inv;
  r.wb = eb * inv;
  return r;
}

__global__ void __launch_bounds__(256) lse_merge_f32_kernel(long long n_vec, int vec_per_head,
                                                            const float4 *oa,
                                                            const float *__restrict__ la,
                                                            const float4 *ob,
                                                            const float *__restrict__ lb, float4 *oo,
                                                            float *lo) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n_vec;
       i += (long long)gridDim.x * blockDim.x) {
    const long long rh = i / vec_per_head;
    const MergeW w = merge_weights(__ldg(la + rh), __ldg(lb + rh));
    const float4 a = __ldcs(oa + i), b = __ldcs(ob + i);
    float4 r;
    r.x = w.wa * a.x + w.wb * b.x;
    r.y = w.wa * a.y + w.wb * b.y;
    r.z = w.wa * a.z + w.wb * b.z;
    r.w = w.wa * a.w + w.wb * b.w;
    __stcs(oo + i, r);
    if (i - rh * vec_per_head == 0) lo[rh] = w.L;
  }
}

__global__ void __launch_bounds__(256) lse_merge_bf16_kernel(long long n_vec, int vec_per_head,
                                                             const uint4 *oa,
                                                             const float *__restrict__ la,
                                                             const uint4 *ob,
                                                             const float *__restrict__ lb, uint4 *oo,
                                                             float *lo) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n_vec;
       i += (long long)gridDim.x * blockDim.x) {
    const long long rh = i / vec_per_head;
    const MergeW w = merge_weights(__ldg(la + rh), __ldg(lb + rh));
    uint4 a = __ldcs(oa + i), b = __ldcs(ob + i), r;
    const uint32_t *pa = reinterpret_cast<const uint32_t *>(&a);
    const uint32_t *pb = reinterpret_cast<const uint32_t *>(&b);
    uint32_t *pr = reinterpret_cast<uint32_t *>(&r);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(pa + j));
      const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(pb + j));
      pr[j] = pack_bf16x2(w.wa * fa.x + w.wb * fb.x, w.wa * fa.y + w.wb * fb.y);
    }
    __stcs(oo + i, r);
    if (i - rh * vec_per_head == 0) lo[rh] = w.L;
  }
}

static int stream_grid(long long n_threads, int block) {
  const long long want = (n_threads + block - 1) / block;
  const long long cap = (long long)sm_count() * 8;  // 8 x 256 threads resident per SM
  return (int)(want < cap ? (want < 1 ? 1 : want) : cap);
}

ispa_status launch_lse_merge(int rows, int H, int d, ispa_dtype dt, const void *oa, const float *la,
                             const void *ob, const float *lb, void *oo, float *lo, cudaStream_t s) {
  const int per_vec = dt == ISPA_F32 ? 4 : 8;
  const int vph = d / per_vec;
  const long long n_vec = (long long)rows * H * vph;
  if (n_vec == 0) return ISPA_OK;
  const int grid = stream_grid(n_vec, 256);
  if (dt == ISPA_F32)
    lse_merge_f32_kernel<<<grid, 256, 0, s>>>(n_vec, vph, (const float4 *)oa, la, (const float4 *)ob, lb,
                                              (float4 *)oo, lo);
  else
    lse_merge_bf16_kernel<<<grid, 256, 0, s>>>(n_vec, vph, (const uint4 *)oa, la, (const uint4 *)ob, lb,
                                               (uint4 *)oo, lo);
  note_launch();
  return cuda_status(cudaGetLastError(), "lse_merge launch");
}

// ---------------------------------------------------------------------------
// W_new = W + dW  (4 elements per thread; D * Dout % 4 == 0 is checked by the caller)
// ---------------------------------------------------------------------------
template <typename TW, typename TO>
__global__ void __launch_bounds__(256) absorb_weight_kernel(long long n4, const TW *__restrict__ W,
                                                            const float4 *__restrict__ dW, TO *Wn) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4;
       i += (long long)gridDim.x * blockDim.x) {
    const float4 d = __ldg(dW + i);
    float w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) w[j] = load_as_float(W + 4 * i + j);
    const float r[4] = {w[0] + d.x, w[1] + d.y, w[2] + d.z, w[3] + d.w};
    if constexpr (sizeof(TO) == 4) {
      reinterpret_cast<float4 *>(Wn)[i] = make_float4(r[0], r[1], r[2], r[3]);
    } else {
      uint2 p;
      p.x = pack_bf16x2(r[0], r[1]);
      p.y = pack_bf16x2(r[2], r[3]);
      reinterpret_cast<uint2 *>(Wn)[i] = p;
    }
  }
}

ispa_status launch_absorb_weight(int D, int Dout, const void *W, ispa_dtype wdt, const float *dW, void *Wn,
                                 ispa_dtype odt, cudaStream_t s) {
  const long long n4 = (long long)D * Dout / 4;
  if (n4 == 0) return ISPA_OK;
  const int grid = stream_grid(n4, 256);
  const float4 *d4 = reinterpret_cast<const float4 *>(dW);
  if (wdt == ISPA_F32 && odt == ISPA_F32)
    absorb_weight_kernel<float, float><<<grid, 256, 0, s>>>(n4, (const float *)W, d4, (float *)Wn);
  else if (wdt == ISPA_F32)
    absorb_weight_kernel<float, __nv_bfloat16><<<grid, 256, 0, s>>>(n4, (const float *)W, d4,
                                                                   (__nv_bfloat16 *)Wn);
  else if (odt == ISPA_F32)
    absorb_weight_kernel<__nv_bfloat16, float><<<grid, 256, 0, s>>>(n4, (const __nv_bfloat16 *)W, d4,
                                                                   (float *)Wn);
  else
    absorb_weight_kernel<__nv_bfloat16, __nv_bfloat16>
        <<<grid, 256, 0, s>>>(n4, (const __nv_bfloat16 *)W, d4, (__nv_bfloat16 *)Wn);
  note_launch();
  return cuda_status(cudaGetLastError(), "absorb_weight launch");
}

// ---------------------------------------------------------------------------
// Layer selection: rank_i = #{j : (eps_j, j) < (eps_i, i)} with NaN after every
// number; layer i is chosen iff rank_i < K; idx lists chosen layers ascending.
// One CTA; N <= 4096 layers, O(N^2 / threads) comparisons.
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool eps_before(double a, int i, double b, int j) {
  const bool na = a != a, nb = b != b;
  if (na || nb) return (na == nb) ? i < j : nb;
  return a < b || (a == b && i < j);
}

__global__ void __launch_bounds__(1024) select_kernel(int N, const double *__restrict__ eps, int K,
                                                      unsigned char *is_local, int *idx) {
  __shared__ double s_eps[4096];
  __shared__ unsigned char s_sel[4096];
  for (int i = threadIdx.x; i < N; i += blockDim.x) s_eps[i] = eps[i];
  __syncthreads();
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    const double e = s_eps[i];
    int rank = 0;
    for (int j = 0; j < N; ++j) rank += eps_before(s_eps[j], j, e, i) ? 1 : 0;
    s_sel[i] = rank < K ? 1 : 0;
    is_local[i] = s_sel[i];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    if (!s_sel[i]) continue;
    int pos = 0;
    for (int j = 0; j < i; ++j) pos += s_sel[j];
    idx[pos] = i;
  }
}

ispa_status launch_select(int N, const double *eps, int K, unsigned char *is_local, int *idx, cudaStream_t s) {
  if (N == 0) return ISPA_OK;
  select_kernel<<<1, 1024, 0, s>>>(N, eps, K, is_local, idx);
  note_launch();
  return cuda_status(cudaGetLastError(), "select launch");
}

// ---------------------------------------------------------------------------
// KV eviction of an L-layer and its inverse: the kept token rows of every
// instance, back to back in the compact layout; 16 bytes per thread and
// iteration.  Compact row r of an instance is full row b0 + r for r < len0,
// b1 + r - len0 after.  gather: compact <- full; otherwise full <- compact.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) kv_remap_kernel(int B, long long full_rows, long long kept_rows, long long b0,
                                                       long long len0, long long b1, int vec_per_row, int gather,
                                                       const uint4 *__restrict__ k, const uint4 *__restrict__ v,
                                                       uint4 *__restrict__ ko, uint4 *__restrict__ vo) {
  const long long per_inst = kept_rows * vec_per_row;
  const long long n = (long long)B * per_inst;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
    const long long b = e / per_inst, rem = e - b * per_inst;
    const long long r = rem / vec_per_row, c = rem - r * vec_per_row;
    const long long fr = r < len0 ? b0 + r : b1 + (r - len0);
    const long long fi = (b * full_rows + fr) * vec_per_row + c;
    if (gather) {
      ko[e] = k[fi];
      vo[e] = v[fi];
    } else {
      ko[fi] = k[e];
      vo[fi] = v[e];
    }
  }
}

ispa_status launch_kv_remap(int B, long long full_rows, long long kept_rows, long long b0, long long len0,
                            long long b1, long long row_bytes, bool gather, const void *k, const void *v,
                            void *k_out, void *v_out, cudaStream_t s) {
  if (B == 0 || kept_rows == 0) return ISPA_OK;
  kv_remap_kernel<<<sm_count() * 4, 256, 0, s>>>(B, full_rows, kept_rows, b0, len0, b1, (int)(row_bytes / 16),
                                                gather ? 1 : 0, (const uint4 *)k, (const uint4 *)v, (uint4 *)k_out,
                                                (uint4 *)v_out);
  note_launch();
  return cuda_status(cudaGetLastError(), "kv remap launch");
}

// ---------------------------------------------------------------------------
// Failure-detection self-test: the bounded wait of the kernels, on a barrier
// that no arrival completes, so that it runs out and reports.
// ---------------------------------------------------------------------------
__global__ void selftest_wait_kernel(DevErr e) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) wait_parity(&bar, 0, e, &abort_flag, ISPA_SELFTEST_SITE);
}

ispa_status launch_selftest_wait(const DevErr &e, cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>(e);
  note_launch();
  return cuda_status(cudaGetLastError(), "self-test launch");
}

}  // namespace ispa
