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
  const float *v_unscale;  // [B * H]: 2^-s of the fp16 copy of V (see prepare_v)
  void *o_loc, *o_hist, *o_full;
  float *l_loc, *l_hist, *l_full;
  DevErr err;
};

// ---------------------------------------------------------------------------
// fp16 copy of V.  P = exp(S - m) is rounded to 16 bits before the PV product;
// in fp16 (11 significant bits) that rounding is 8x finer than in bf16, which
// keeps the output error well inside the parity tolerance.  tcgen05 kind::f16
// needs both operands in the same type, so V is converted once per call:
// each head of each instance is scaled by a power of two 2^s so that its
// largest |v| lies in [2^14, 2^15) (exact in fp16, far from overflow), and the
// epilogue multiplies O by 2^-s (exact).  Only the rows the tiles read are
// converted: every range rounded up to whole 128-row tiles.
// ---------------------------------------------------------------------------
struct VPrep {
  int B, H, Lkv;
  int n_ext;
  int ext_begin[3], ext_end[3];  // row extents the tiles touch
};

// Per-(instance, head) max |v|.  Each thread keeps one 16-byte column group c8
// (8 values of one head) and walks rows; the 16 lanes that cover one head
// combine by shuffles and one lane per head issues the atomic.
__global__ void __launch_bounds__(256) v_amax_kernel(VPrep p, const __nv_bfloat16 *__restrict__ v,
                                                     unsigned int *amax_bits) {
  const int D = p.H * kD;
  const int vec_per_row = D / 8;                       // multiple of 16 (kD / 8 = 16 per head)
  const int b = blockIdx.y;
  const int lanes = gridDim.x * blockDim.x;
  const int row_step = lanes / vec_per_row;            // rows advanced per pass (>= 1 by the launch)
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  const int c8 = tid % vec_per_row;
  const int r0 = tid / vec_per_row;
  float m = 0.f;
  if (r0 < row_step) {
    for (int e = 0; e < p.n_ext; ++e)
      for (int row = p.ext_begin[e] + r0; row < p.ext_end[e]; row += row_step) {
        const uint4 in = __ldg(reinterpret_cast<const uint4 *>(v + ((long long)b * p.Lkv + row) * D) + c8);
        const uint32_t w[4] = {in.x, in.y, in.z, in.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[j]));
          m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
      }
  }
  // vec_per_row = 16 H and warps start at multiples of 32, so lanes 16k..16k+15
  // hold the 16 column groups of one head of one row: reduce them by shuffles.
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 15) == 0 && r0 < row_step) atomicMax(amax_bits + b * p.H + (c8 * 8) / kD, __float_as_uint(m));
}

__device__ __forceinline__ int v_exponent(unsigned int amax_bits) {
  const float a = __uint_as_float(amax_bits);
  if (!(a > 0.f) || !isfinite(a)) return 0;
  return 14 - ilogbf(a);  // a * 2^s in [2^14, 2^15)
}

__global__ void __launch_bounds__(256) v_to_f16_kernel(VPrep p, const __nv_bfloat16 *__restrict__ v,
                                                       const unsigned int *__restrict__ amax_bits, __half *v16,
                                                       float *v_unscale) {
  const int D = p.H * kD;
  const int vec_per_row = D / 8;
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < p.B * p.H; i += blockDim.x) v_unscale[i] = ldexpf(1.f, -v_exponent(amax_bits[i]));
  for (int e = 0; e < p.n_ext; ++e) {
    const long long rows = p.ext_end[e] - p.ext_begin[e];
    const long long n = (long long)p.B * rows * vec_per_row;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
      const int c8 = (int)(i % vec_per_row);
      const long long br = i / vec_per_row;
      const int b = (int)(br / rows);
      const long long row = p.ext_begin[e] + br % rows;
      const int h = (c8 * 8) / kD;
      const float scale = ldexpf(1.f, v_exponent(amax_bits[b * p.H + h]));
      const long long off = ((long long)b * p.Lkv + row) * D + c8 * 8;
      const uint4 in = *reinterpret_cast<const uint4 *>(v + off);
      const uint32_t w[4] = {in.x, in.y, in.z, in.w};
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[j]));
        const float lo = fminf(fmaxf(f.x * scale, -65504.f), 65504.f);
        const float hi = fminf(fmaxf(f.y * scale, -65504.f), 65504.f);
        __half2 hh = __floats2half2_rn(lo, hi);
        o[j] = *reinterpret_cast<uint32_t *>(&hh);
      }
      *reinterpret_cast<uint4 *>(v16 + off) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

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
      const uint32_t idesc_pv = make_idesc(128, 128, 0, 0, 1);  // fp16 P (TMEM) x fp16 V (smem)
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
      // row maximum with 8 independent partial maxima (no 128-long dependency chain)
      float mx[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) mx[t] = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        if (c >= n_valid) s[c] = -INFINITY;
        mx[c & 7] = fmaxf(mx[c & 7], s[c]);
      }
      float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
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
      // P = exp2(s * scale * log2e - m_ref) <= 2^8, packed to fp16 pairs into TMEM P[j % 2].
      const float neg_m = -m_ref;
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const float p0 = ex2(fmaf(s[c * 32 + 2 * t], P.scale_log2, neg_m));
          const float p1 = ex2(fmaf(s[c * 32 + 2 * t + 1], P.scale_log2, neg_m));
          ls[t & 3] += p0 + p1;
          pk[t] = pack_f16x2(p0, p1);
        }
        tmem_st16(lane_base + kColP0 + (uint32_t)(j & 1) * 64 + c * 16, pk);
      }
      tmem_wait_st();
      l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
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
      const float inv_l = P.v_unscale[b * P.H + h] / l;  // undoes the power-of-two scaling of V too
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

ispa_status map3d_16(CUtensorMap *m, const void *base, int D, int rows, int B, CUtensorMapDataType dt) {
  const uint64_t dims[3] = {(uint64_t)D, (uint64_t)rows, (uint64_t)B};
  const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)D * 2 * (uint64_t)rows};
  const uint32_t box[3] = {64, 128, 1};
  return make_tmap(m, dt, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

size_t attn_tc_workspace_bytes(int B, int H, int Lkv) {
  return a256((size_t)B * Lkv * H * kD * 2) + 2 * a256((size_t)B * H * 4);
}

ispa_status launch_attn_tc(const ispa_attn_desc &d, const GroupRanges &g, float scale, const void *q,
                           const void *k, const void *v, void *o_loc, float *l_loc, void *o_hist, float *l_hist,
                           void *o_full, float *l_full, void *workspace, cudaStream_t s) {
  if (g.Lq == 0) return ISPA_OK;
  AttnParams P{};
  ispa_status st = device_err(&P.err);
  if (st != ISPA_OK) return st;
  const int D = d.H * kD;

  // ---- fp16 copy of the V rows the tiles read (workspace)
  char *ws = static_cast<char *>(workspace);
  __half *v16 = reinterpret_cast<__half *>(ws);
  unsigned int *amax = reinterpret_cast<unsigned int *>(ws + a256((size_t)d.B * g.Lkv * D * 2));
  float *v_unscale = reinterpret_cast<float *>(ws + a256((size_t)d.B * g.Lkv * D * 2) + a256((size_t)d.B * d.H * 4));
  VPrep vp{};
  vp.B = d.B;
  vp.H = d.H;
  vp.Lkv = g.Lkv;
  auto add_ext = [&](int beg, int end) {
    if (end <= beg) return;
    const int tiles = (end - beg + kTileK - 1) / kTileK;
    vp.ext_begin[vp.n_ext] = beg;
    vp.ext_end[vp.n_ext] = min(g.Lkv, beg + tiles * kTileK);
    ++vp.n_ext;
  };
  for (int r = 0; r < g.n_loc; ++r) add_ext(g.loc_begin[r], g.loc_end[r]);
  add_ext(g.hist_begin, g.hist_end);
  cudaError_t e = cudaMemsetAsync(amax, 0, (size_t)d.B * d.H * 4, s);
  if (e != cudaSuccess) return cuda_status(e, "attention workspace clear");
  const int vec_per_row = D / 8;
  const int amax_blocks = max((vec_per_row + 255) / 256, (sm_count() * 8 + d.B - 1) / d.B);
  v_amax_kernel<<<dim3(amax_blocks, d.B), 256, 0, s>>>(vp, static_cast<const __nv_bfloat16 *>(v), amax);
  v_to_f16_kernel<<<sm_count() * 8, 256, 0, s>>>(vp, static_cast<const __nv_bfloat16 *>(v), amax, v16, v_unscale);
  note_launch(2);
  if ((st = cuda_status(cudaGetLastError(), "V conversion launch")) != ISPA_OK) return st;
  P.v_unscale = v_unscale;

  CUtensorMap tq, tk, tv;
  if ((st = map3d_16(&tq, q, D, g.Lq, d.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16)) != ISPA_OK) return st;
  if ((st = map3d_16(&tk, k, D, g.Lkv, d.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16)) != ISPA_OK) return st;
  if ((st = map3d_16(&tv, v16, D, g.Lkv, d.B, CU_TENSOR_MAP_DATA_TYPE_FLOAT16)) != ISPA_OK) return st;
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
