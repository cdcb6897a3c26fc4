// attn_simt.cu -- two-group attention on fp32 inputs with fp32 CUDA-core arithmetic.
//
// The fp32 path keeps full fp32 accuracy (tcgen05 has no fp32 MMA kind).  One
// warp owns one query row of one head; a CTA of 8 warps shares 32-key K/V
// tiles staged in shared memory.  Within a tile lane j scores key j (a full
// d-long dot product), the warp forms the tile's softmax weights with
// shuffles, and every lane accumulates its d/32 output dimensions.  Each
// group keeps its own online-softmax state (running max m, sum l, output o);
// at the end of a group the kernel writes O = o / l and L = m + log l, and
// with the fused merge it combines both groups by their LSE.
#include "internal.h"

namespace ispa {

namespace {

constexpr int kWarps = 8;
constexpr int kKeys = 32;

template <int D>
struct GroupState {
  float m, l;
  float o[D / 32];
  __device__ void reset() {
    m = -INFINITY;
    l = 0.f;
#pragma unroll
    for (int i = 0; i < D / 32; ++i) o[i] = 0.f;
  }
};

// Folds one staged tile (n_valid keys) into the state of this warp's query.
template <int D>
__device__ __forceinline__ void fold_tile(GroupState<D> &st, const float *qs, const float *ks, const float *vs,
                                          int n_valid, float scale, int lane) {
  float s = -INFINITY;
  if (lane < n_valid) {
    const float *kr = ks + lane * (D + 1);
    float acc = 0.f;
#pragma unroll 8
    for (int t = 0; t < D; ++t) acc = fmaf(qs[t], kr[t], acc);
    s = acc * scale;
  }
  const float tmax = warp_max(s);
  const float m_new = fmaxf(st.m, tmax);
  const float p = (lane < n_valid) ? expf(s - m_new) : 0.f;
  const float corr = (st.m == -INFINITY) ? 0.f : expf(st.m - m_new);
  st.l = st.l * corr + warp_sum(p);
  st.m = m_new;
#pragma unroll
  for (int i = 0; i < D / 32; ++i) st.o[i] *= corr;
  for (int j = 0; j < n_valid; ++j) {
    const float pj = __shfl_sync(0xffffffffu, p, j);
    const float *vr = vs + j * (D + 1);
#pragma unroll
    for (int i = 0; i < D / 32; ++i) st.o[i] = fmaf(pj, vr[lane + 32 * i], st.o[i]);
  }
}

template <typename TO>
__device__ __forceinline__ void store_out(TO *p, float x);
template <>
__device__ __forceinline__ void store_out<float>(float *p, float x) { *p = x; }
template <>
__device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

template <int D, typename TO>
__device__ __forceinline__ void write_group(const GroupState<D> &st, TO *o, float *lse, long long o_off,
                                            long long l_off, int lane, float *o_norm) {
  const bool empty = st.l == 0.f;
  const float inv = empty ? 0.f : 1.f / st.l;
#pragma unroll
  for (int i = 0; i < D / 32; ++i) {
    o_norm[i] = st.o[i] * inv;
    if (o) store_out(o + o_off + lane + 32 * i, o_norm[i]);
  }
  if (lse && lane == 0) lse[l_off] = empty ? -INFINITY : st.m + logf(st.l);
}

template <int D, typename TO>
__global__ void __launch_bounds__(kWarps * 32) attn_simt_kernel(GroupRanges g, int H, float scale,
                                                                const float *__restrict__ q,
                                                                const float *__restrict__ k,
                                                                const float *__restrict__ v, TO *o_loc,
                                                                float *l_loc, TO *o_hist, float *l_hist,
                                                                TO *o_full, float *l_full) {
  __shared__ float ks[kKeys * (D + 1)];
  __shared__ float vs[kKeys * (D + 1)];
  __shared__ float qs[kWarps][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int row = blockIdx.x * kWarps + warp;
  const bool active = row < g.Lq;
  const long long head_stride = (long long)H * D;
  if (active)
    for (int t = lane; t < D; t += 32) qs[warp][t] = q[((long long)b * g.Lq + row) * head_stride + h * D + t];

  GroupState<D> st;
  float o_loc_n[D / 32], o_hist_n[D / 32];
  float L_loc = -INFINITY, L_hist = -INFINITY;
  const long long o_off = ((long long)b * g.Lq + row) * head_stride + h * D;
  const long long l_off = ((long long)b * g.Lq + row) * H + h;
  const float *kb = k + (long long)b * g.Lkv * head_stride + h * D;
  const float *vb = v + (long long)b * g.Lkv * head_stride + h * D;

  for (int grp = 0; grp < 2; ++grp) {
    st.reset();
    const int n_ranges = grp == 0 ? g.n_loc : (g.hist_end > g.hist_begin ? 1 : 0);
    for (int r = 0; r < n_ranges; ++r) {
      const int beg = grp == 0 ? g.loc_begin[r] : g.hist_begin;
      const int end = grp == 0 ? g.loc_end[r] : g.hist_end;
      for (int t0 = beg; t0 < end; t0 += kKeys) {
        const int n_valid = min(kKeys, end - t0);
        __syncthreads();
        for (int e = threadIdx.x; e < n_valid * D; e += blockDim.x) {
          const int kr = e / D, kc = e - kr * D;
          ks[kr * (D + 1) + kc] = kb[(long long)(t0 + kr) * head_stride + kc];
          vs[kr * (D + 1) + kc] = vb[(long long)(t0 + kr) * head_stride + kc];
        }
        __syncthreads();
        if (active) fold_tile<D>(st, qs[warp], ks, vs, n_valid, scale, lane);
      }
    }
    if (!active) continue;
    if (grp == 0) {
      write_group<D, TO>(st, o_loc, l_loc, o_off, l_off, lane, o_loc_n);
      L_loc = st.l == 0.f ? -INFINITY : st.m + logf(st.l);
    } else {
      write_group<D, TO>(st, o_hist, l_hist, o_off, l_off, lane, o_hist_n);
      L_hist = st.l == 0.f ? -INFINITY : st.m + logf(st.l);
    }
  }
  if (!active || !o_full) return;
  const float m = fmaxf(L_loc, L_hist);
  float wa = 0.f, wb = 0.f, L = -INFINITY;
  if (m != -INFINITY) {
    const float ea = expf(L_loc - m), eb = expf(L_hist - m), s = ea + eb;
    wa = ea / s;
    wb = eb / s;
    L = m + logf(s);
  }
#pragma unroll
  for (int i = 0; i < D / 32; ++i) store_out(o_full + o_off + lane + 32 * i, wa * o_loc_n[i] + wb * o_hist_n[i]);
  if (lane == 0) l_full[l_off] = L;
}

template <int D, typename TO>
ispa_status launch_d(const ispa_attn_desc &d, const GroupRanges &g, float scale, const float *q, const float *k,
                     const float *v, void *o_loc, float *l_loc, void *o_hist, float *l_hist, void *o_full,
                     float *l_full, cudaStream_t s) {
  dim3 grid((g.Lq + kWarps - 1) / kWarps, d.H, d.B);
  attn_simt_kernel<D, TO><<<grid, kWarps * 32, 0, s>>>(g, d.H, scale, q, k, v, (TO *)o_loc, l_loc,
                                                       (TO *)o_hist, l_hist, (TO *)o_full, l_full);
  note_launch();
  return cuda_status(cudaGetLastError(), "attn_simt launch");
}

}  // namespace

ispa_status launch_attn_simt(const ispa_attn_desc &d, const GroupRanges &g, float scale, const float *q,
                             const float *k, const float *v, void *o_loc, float *l_loc, void *o_hist,
                             float *l_hist, void *o_full, float *l_full, cudaStream_t s) {
  if (g.Lq == 0) return ISPA_OK;
  const bool bf = d.out_dtype == ISPA_BF16;
  switch (d.head_dim) {
    case 32:
      return bf ? launch_d<32, __nv_bfloat16>(d, g, scale, q, k, v, o_loc, l_loc, o_hist, l_hist, o_full, l_full, s)
                : launch_d<32, float>(d, g, scale, q, k, v, o_loc, l_loc, o_hist, l_hist, o_full, l_full, s);
    case 64:
      return bf ? launch_d<64, __nv_bfloat16>(d, g, scale, q, k, v, o_loc, l_loc, o_hist, l_hist, o_full, l_full, s)
                : launch_d<64, float>(d, g, scale, q, k, v, o_loc, l_loc, o_hist, l_hist, o_full, l_full, s);
    default:
      return bf ? launch_d<128, __nv_bfloat16>(d, g, scale, q, k, v, o_loc, l_loc, o_hist, l_hist, o_full, l_full, s)
                : launch_d<128, float>(d, g, scale, q, k, v, o_loc, l_loc, o_hist, l_hist, o_full, l_full, s);
  }
}

}  // namespace ispa
