// attn_tc.cu -- two-group attention on tcgen05 tensor cores (bf16 in, fp32 accumulate, d = 128).
//
// One CTA computes one 128-query tile of one head of one instance and walks the
// KV tiles of the local group (sink range, then current range) followed by the
// history group.  Each group keeps its own online-softmax state; at the end of
// a group the normalised output and its log-sum-exp are written, and after the
// history group the optional fused merge combines both groups by their LSE.
//
// Warp roles (192 threads, one CTA per SM):
//   warp 0      TMA producer: Q once, then K and V tiles (128 keys x 128 dims)
//               through two-stage rings with separate K and V barriers.
//   warp 1      TMEM allocator and MMA issuer:
//                 S_j = Q K_j^T       -> TMEM S[j % 2]   (A, B from shared memory)
//                 O  += P_j V_j       -> TMEM O          (A = P from TMEM, B = V)
//               issue order S_0, S_1, PV_0, S_2, PV_1, ... so that the
//               softmax of tile j overlaps the MMAs of tiles j+1 and j-1.
//   warps 2..5  softmax / correction / epilogue, one query row per thread
//               (TMEM lane = row).  P_j is written as packed bf16 to TMEM
//               P[j % 2] (K/2 32-bit columns per row).  The running maximum is
//               only moved (and O rescaled) when a row's tile maximum exceeds
//               it by more than 2^8, so O is rarely touched off the MMA path.
//
// TMEM columns: S0 [0,128) S1 [128,256) O [256,384) P0 [384,448) P1 [448,512).
//
// Ordering argument (every TMEM buffer has one writer at a time):
//   * S_j overwrites S[j%2] only after P_{j-2} was published, i.e. after the
//     softmax of tile j-2 finished its tcgen05.ld of that buffer.
//   * The softmax of tile j writes P[j%2] after S_j completed; S_j's commit
//     covers every earlier MMA, including PV_{j-2} which read P[j%2].
//   * O is rescaled by the softmax of tile j only after PV_{j-1} completed
//     (o_done) and before PV_j is issued (PV_j waits for P_j).
//   * At the end of the local group the epilogue reads O after PV of that tile
//     and releases it (o_free) before the first history PV overwrites it.
#include "internal.h"

namespace ispa {

namespace {

constexpr int kThreads = 192;
constexpr int kTileQ = 128, kTileK = 128, kD = 128;
constexpr int kBoxBytes = 128 * 128;          // 128 rows x 64 bf16
constexpr int kTileBytes = 2 * kBoxBytes;     // 128 rows x 128 bf16
constexpr int kStages = 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColO = 256, kColP0 = 384;
constexpr float kRescaleThreshold = 8.0f;     // log2 units

struct AttnParams {
  int H, Lq, q_tiles;
  int n_ranges;            // ranges 0..n_ranges-1; the first n_loc_ranges are local
  int n_loc_ranges;
  int r_begin[3], r_end[3];
  int n_loc_tiles, n_tiles;
  float scale_log2;        // softmax scale * log2(e)
  void *o_loc, *o_hist, *o_full;
  float *l_loc, *l_hist, *l_full;
  DevErr err;
};

struct SmemLayout {
  uint8_t q[kTileBytes];
  uint8_t k[kStages][kTileBytes];
  uint8_t v[kStages][kTileBytes];
  uint64_t q_full;
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t v_full[kStages], v_empty[kStages];
  uint64_t s_full[2], p_full[2];
  uint64_t o_done, o_free, drain;
  uint32_t tmem_base;
  int abort;
};

constexpr int kSmemBytes = sizeof(SmemLayout) + 1024;

// Walks the tile sequence: local ranges first, then history.
struct TileIter {
  int range, t0;
  __device__ void start(const AttnParams &P) {
    range = 0;
    t0 = P.n_ranges > 0 ? P.r_begin[0] : 0;
  }
  __device__ int valid(const AttnParams &P) const { return min(kTileK, P.r_end[range] - t0); }
  __device__ void next(const AttnParams &P) {
    t0 += kTileK;
    if (t0 >= P.r_end[range]) {
      ++range;
      if (range < P.n_ranges) t0 = P.r_begin[range];
    }
  }
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <typename TO>
__device__ __forceinline__ void store_row32(TO *dst, const float (&x)[32]);
template <>
__device__ __forceinline__ void store_row32<float>(float *dst, const float (&x)[32]) {
  float4 *d4 = reinterpret_cast<float4 *>(dst);
#pragma unroll
  for (int v = 0; v < 8; ++v) d4[v] = make_float4(x[4 * v], x[4 * v + 1], x[4 * v + 2], x[4 * v + 3]);
}
template <>
__device__ __forceinline__ void store_row32<__nv_bfloat16>(__nv_bfloat16 *dst, const float (&x)[32]) {
  uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
  for (int v = 0; v < 4; ++v)
    d4[v] = make_uint4(pack_bf16x2(x[8 * v], x[8 * v + 1]), pack_bf16x2(x[8 * v + 2], x[8 * v + 3]),
                       pack_bf16x2(x[8 * v + 4], x[8 * v + 5]), pack_bf16x2(x[8 * v + 6], x[8 * v + 7]));
}

template <typename TO>
__device__ __forceinline__ void load_row32(const TO *src, float (&x)[32]);
template <>
__device__ __forceinline__ void load_row32<float>(const float *src, float (&x)[32]) {
  const float4 *s4 = reinterpret_cast<const float4 *>(src);
#pragma unroll
  for (int v = 0; v < 8; ++v) {
    const float4 t = s4[v];
    x[4 * v] = t.x;
    x[4 * v + 1] = t.y;
    x[4 * v + 2] = t.z;
    x[4 * v + 3] = t.w;
  }
}
template <>
__device__ __forceinline__ void load_row32<__nv_bfloat16>(const __nv_bfloat16 *src, float (&x)[32]) {
  const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const uint4 t = s4[v];
    const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
      x[8 * v + 2 * i] = f.x;
      x[8 * v + 2 * i + 1] = f.y;
    }
  }
}

template <typename TO>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                   const __grid_constant__ CUtensorMap tv, AttnParams P) {
  extern __shared__ uint8_t smem_raw[];
  SmemLayout &sm =
      *reinterpret_cast<SmemLayout *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  volatile int *abort = &sm.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x % P.q_tiles;
  const int h = blockIdx.x / P.q_tiles;
  const int b = blockIdx.y;
  const int q0 = qt * kTileQ;
  const bool has_hist = P.n_tiles > P.n_loc_tiles;

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.p_full[s], 128);
    }
    mbar_init(&sm.o_done, 1);
    mbar_init(&sm.o_free, 128);
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
  }
  if (warp == 1) tmem_alloc(&sm.tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const int x0 = h * kD;
      mbar_arrive_expect_tx(&sm.q_full, kTileBytes);
      tma_load_3d(sm.q, &tq, &sm.q_full, x0, q0, b);
      tma_load_3d(sm.q + kBoxBytes, &tq, &sm.q_full, x0 + 64, q0, b);
      uint32_t k_pend = 0, v_pend = 0, k_ph = 0, v_ph = 0;
      TileIter it;
      it.start(P);
      for (int j = 0; j < P.n_tiles; ++j, it.next(P)) {
        const int s = j % kStages;
        const uint32_t ph = (j / kStages) & 1;
        if (!wait_parity(&sm.k_empty[s], ph ^ 1, P.err, abort, 11)) break;
        mbar_arrive_expect_tx(&sm.k_full[s], kTileBytes);
        tma_load_3d(sm.k[s], &tk, &sm.k_full[s], x0, it.t0, b);
        tma_load_3d(sm.k[s] + kBoxBytes, &tk, &sm.k_full[s], x0 + 64, it.t0, b);
        k_pend |= 1u << s;
        k_ph = (k_ph & ~(1u << s)) | (ph << s);
        if (!wait_parity(&sm.v_empty[s], ph ^ 1, P.err, abort, 12)) break;
        mbar_arrive_expect_tx(&sm.v_full[s], kTileBytes);
        tma_load_3d(sm.v[s], &tv, &sm.v_full[s], x0, it.t0, b);
        tma_load_3d(sm.v[s] + kBoxBytes, &tv, &sm.v_full[s], x0 + 64, it.t0, b);
        v_pend |= 1u << s;
        v_ph = (v_ph & ~(1u << s)) | (ph << s);
      }
      if (*abort) {  // let copies in flight land before the CTA exits
        wait_parity_drain(&sm.q_full, 0, P.err);
        for (int s = 0; s < kStages; ++s) {
          if (k_pend & (1u << s)) wait_parity_drain(&sm.k_full[s], (k_ph >> s) & 1, P.err);
          if (v_pend & (1u << s)) wait_parity_drain(&sm.v_full[s], (v_ph >> s) & 1, P.err);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = make_idesc(128, 128, 1, 0, 0);
      const uint32_t idesc_pv = make_idesc(128, 128, 1, 0, 1);
      const uint32_t q_addr = smem_u32(sm.q);
      bool ok = wait_parity(&sm.q_full, 0, P.err, abort, 21);
      for (int j = 0; ok && j <= P.n_tiles; ++j) {
        if (j < P.n_tiles) {
          const int s = j % kStages;
          if (!wait_parity(&sm.k_full[s], (j / kStages) & 1, P.err, abort, 22)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sm.k[s]);
          const uint32_t d_s = tmem + kColS0 + (uint32_t)(j & 1) * 128;
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint32_t off = (uint32_t)(kk >> 2) * kBoxBytes + (uint32_t)(kk & 3) * 32;
            mma_ss(d_s, smem_desc_sw128(q_addr + off, 16, 1024), smem_desc_sw128(k_addr + off, 16, 1024), idesc_qk,
                   kk > 0 ? 1u : 0u, 0);
          }
          mma_commit(&sm.k_empty[s]);
          mma_commit(&sm.s_full[j & 1]);
        }
        if (j >= 1) {
          const int i = j - 1;
          const int s = i % kStages;
          if (!wait_parity(&sm.p_full[i & 1], (i >> 1) & 1, P.err, abort, 23)) {
            ok = false;
            break;
          }
          if (i == P.n_loc_tiles && !wait_parity(&sm.o_free, 0, P.err, abort, 24)) {
            ok = false;
            break;
          }
          if (!wait_parity(&sm.v_full[s], (i / kStages) & 1, P.err, abort, 25)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const bool first = (i == 0) || (i == P.n_loc_tiles);
          const uint32_t v_addr = smem_u32(sm.v[s]);
          const uint32_t a_p = tmem + kColP0 + (uint32_t)(i & 1) * 64;
#pragma unroll
          for (int kk = 0; kk < kTileK / 16; ++kk) {
            mma_ts(tmem + kColO, a_p + kk * 8, smem_desc_sw128(v_addr + kk * 2048, kBoxBytes, 1024), idesc_pv,
                   (first && kk == 0) ? 0u : 1u);
          }
          mma_commit(&sm.v_empty[s]);
          mma_commit(&sm.o_done);
        }
      }
      if (!ok) {
        mma_commit(&sm.drain);
        wait_parity_drain(&sm.drain, 0, P.err);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // row inside the tile == TMEM lane
    const int qrow = q0 + r;
    const bool row_ok = qrow < P.Lq;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const long long head_row = ((long long)b * P.Lq + (row_ok ? qrow : 0)) * P.H + h;
    TO *o_loc = reinterpret_cast<TO *>(P.o_loc) + head_row * kD;
    TO *o_hist = P.o_hist ? reinterpret_cast<TO *>(P.o_hist) + head_row * kD : nullptr;
    TO *o_full = P.o_full ? reinterpret_cast<TO *>(P.o_full) + head_row * kD : nullptr;
    float m_ref = 0.f, l = 0.f, L_loc = -INFINITY;
    TileIter it;
    it.start(P);
    for (int j = 0; j < P.n_tiles; ++j, it.next(P)) {
      const bool grp_first = (j == 0) || (j == P.n_loc_tiles);
      const bool grp_last = (j == P.n_loc_tiles - 1) || (j == P.n_tiles - 1);
      const int n_valid = it.valid(P);
      bool ok = wait_parity(&sm.s_full[j & 1], (j >> 1) & 1, P.err, abort, 31);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      float s[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t raw[32];
        tmem_ld32(lane_base + kColS0 + (uint32_t)(j & 1) * 128 + c * 32, raw);
        tmem_wait_ld();
#pragma unroll
        for (int t = 0; t < 32; ++t) s[c * 32 + t] = __uint_as_float(raw[t]);
      }
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        if (c >= n_valid) s[c] = -INFINITY;
        mt = fmaxf(mt, s[c]);
      }
      mt *= P.scale_log2;
      if (grp_first) {
        m_ref = mt;
        l = 0.f;
      } else if (__any_sync(0xffffffffu, mt > m_ref + kRescaleThreshold)) {
        // PV_{j-1} must have landed in O before it is rescaled; PV_j waits for P_j.
        ok = wait_parity(&sm.o_done, (uint32_t)((j - 1) & 1), P.err, abort, 32);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after();
        const float m_new = fmaxf(m_ref, mt);
        const float f = ex2(m_ref - m_new);
        m_ref = m_new;
        l *= f;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t o[16];
          tmem_ld16(lane_base + kColO + c * 16, o);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 16; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * f);
          tmem_st16(lane_base + kColO + c * 16, o);
        }
      }
      // P = exp2(s * scale * log2e - m_ref), packed to bf16 pairs into TMEM P[j % 2].
      const float neg_m = -m_ref;
      float lsum = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const float p0 = ex2(fmaf(s[c * 32 + 2 * t], P.scale_log2, neg_m));
          const float p1 = ex2(fmaf(s[c * 32 + 2 * t + 1], P.scale_log2, neg_m));
          lsum += p0 + p1;
          pk[t] = pack_bf16x2(p0, p1);
        }
        tmem_st16(lane_base + kColP0 + (uint32_t)(j & 1) * 64 + c * 16, pk);
      }
      tmem_wait_st();
      l += lsum;
      tc_fence_before();
      mbar_arrive(&sm.p_full[j & 1]);

      if (!grp_last) continue;
      // ---- end of a group: O of this group is complete once PV_j has landed.
      // o_done counts PVs; a parity wait is only exact when the barrier is at
      // most one phase behind, so first wait for PV_{j-1} (PV_{j-2} is covered
      // by the commit of S_j), then for PV_j.
      ok = j == 0 || wait_parity(&sm.o_done, (uint32_t)((j - 1) & 1), P.err, abort, 33);
      ok = ok && wait_parity(&sm.o_done, (uint32_t)(j & 1), P.err, abort, 34);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const bool is_loc = j < P.n_loc_tiles;
      const float inv_l = 1.f / l;
      const float L = (m_ref + log2f(l)) * 0.69314718055994530942f;
      float wa = 1.f, wb = 0.f, L_full = L;
      if (is_loc) {
        L_loc = L;
        if (row_ok) P.l_loc[head_row] = L;
      } else {
        if (row_ok && P.l_hist) P.l_hist[head_row] = L;
        const float mx = fmaxf(L_loc, L);
        const float ea = expf(L_loc - mx), eb = expf(L - mx), se = ea + eb;
        wa = ea / se;
        wb = eb / se;
        L_full = mx + logf(se);
      }
      TO *dst = is_loc ? o_loc : o_hist;
      const bool write_full = o_full != nullptr && (!is_loc || !has_hist);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t raw[32];
        tmem_ld32(lane_base + kColO + c * 32, raw);
        tmem_wait_ld();
        float x[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) x[t] = __uint_as_float(raw[t]) * inv_l;
        if (!row_ok) continue;
        if (dst) store_row32<TO>(dst + c * 32, x);
        if (write_full) {
          if (!is_loc) {
            float y[32];
            load_row32<TO>(o_loc + c * 32, y);
#pragma unroll
            for (int t = 0; t < 32; ++t) x[t] = wa * y[t] + wb * x[t];
          }
          store_row32<TO>(o_full + c * 32, x);
        }
      }
      if (write_full && row_ok) P.l_full[head_row] = L_full;
      if (is_loc && !has_hist && row_ok) {  // empty history group: O = 0, L = -inf
        if (o_hist) {
          const float zero[32] = {};
#pragma unroll 1
          for (int c = 0; c < 4; ++c) store_row32<TO>(o_hist + c * 32, zero);
        }
        if (P.l_hist) P.l_hist[head_row] = -INFINITY;
      }
      if (is_loc && has_hist) {
        tc_fence_before();
        mbar_arrive(&sm.o_free);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

template <typename TO>
ispa_status launch_typed(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv, const AttnParams &P,
                         int B, cudaStream_t s) {
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(attn_tc_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kSmemBytes);
    if (e != cudaSuccess) return cuda_status(e, "attention smem attribute");
    configured_device = dev;
  }
  dim3 grid(P.q_tiles * P.H, B);
  attn_tc_kernel<TO><<<grid, kThreads, kSmemBytes, s>>>(tq, tk, tv, P);
  note_launch();
  return cuda_status(cudaGetLastError(), "tcgen05 attention launch");
}

ispa_status map3d_bf16(CUtensorMap *m, const void *base, int D, int rows, int B) {
  const uint64_t dims[3] = {(uint64_t)D, (uint64_t)rows, (uint64_t)B};
  const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)D * 2 * (uint64_t)rows};
  const uint32_t box[3] = {64, 128, 1};
  return make_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

ispa_status launch_attn_tc(const ispa_attn_desc &d, const GroupRanges &g, float scale, const void *q,
                           const void *k, const void *v, void *o_loc, float *l_loc, void *o_hist, float *l_hist,
                           void *o_full, float *l_full, cudaStream_t s) {
  if (g.Lq == 0) return ISPA_OK;
  AttnParams P{};
  ispa_status st = device_err(&P.err);
  if (st != ISPA_OK) return st;
  const int D = d.H * kD;
  CUtensorMap tq, tk, tv;
  if ((st = map3d_bf16(&tq, q, D, g.Lq, d.B)) != ISPA_OK) return st;
  if ((st = map3d_bf16(&tk, k, D, g.Lkv, d.B)) != ISPA_OK) return st;
  if ((st = map3d_bf16(&tv, v, D, g.Lkv, d.B)) != ISPA_OK) return st;
  P.H = d.H;
  P.Lq = g.Lq;
  P.q_tiles = (g.Lq + kTileQ - 1) / kTileQ;
  P.n_ranges = 0;
  P.n_loc_tiles = 0;
  for (int r = 0; r < g.n_loc; ++r) {
    P.r_begin[P.n_ranges] = g.loc_begin[r];
    P.r_end[P.n_ranges] = g.loc_end[r];
    P.n_loc_tiles += (g.loc_end[r] - g.loc_begin[r] + kTileK - 1) / kTileK;
    ++P.n_ranges;
  }
  P.n_loc_ranges = P.n_ranges;
  P.n_tiles = P.n_loc_tiles;
  if (g.hist_end > g.hist_begin) {
    P.r_begin[P.n_ranges] = g.hist_begin;
    P.r_end[P.n_ranges] = g.hist_end;
    P.n_tiles += (g.hist_end - g.hist_begin + kTileK - 1) / kTileK;
    ++P.n_ranges;
  }
  P.scale_log2 = scale * 1.4426950408889634f;
  P.o_loc = o_loc;
  P.o_hist = o_hist;
  P.o_full = o_full;
  P.l_loc = l_loc;
  P.l_hist = l_hist;
  P.l_full = l_full;
  if (d.out_dtype == ISPA_F32) return launch_typed<float>(tq, tk, tv, P, d.B, s);
  return launch_typed<__nv_bfloat16>(tq, tk, tv, P, d.B, s);
}

}  // namespace ispa
