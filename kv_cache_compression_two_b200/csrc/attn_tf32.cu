// attn_tf32.cu -- two-group attention on fp32 inputs on the tf32 tensor cores, fp32-accurate.
//
// tcgen05 has no fp32 MMA kind; the fp32 workloads use kind::tf32 in three
// passes: every operand x is split into x_hi = the nearest tf32 and
// x_lo = tf32(x - x_hi), and a product a b is a_hi b_hi + a_hi b_lo + a_lo b_hi
// (the dropped a_lo b_lo is below 2^-21 of |a b|), accumulated in fp32 in
// tensor memory [EN-notes, Key Designs 1: each group's normalised output and
// its log-sum-exp].
//
// One CTA computes one 128-query tile of one head of one instance (thread t
// owns query row t, TMEM lane t) and walks 64-key tiles of the local group,
// then of the history group, step by step:
//   1. the 128 threads load the tile's K and V rows, split them and store
//      K (keys x d) and V^T (d x keys) as K-major 128-byte-swizzled operands;
//   2. thread 0 issues S = Q K^T in three passes (Q_hi, Q_lo in TMEM);
//   3. each thread takes its row of S, updates its group's running maximum
//      (rescaling O in TMEM when it grows) and sum, and stores P (hi, lo) as
//      the K-major A operand of the next product;
//   4. thread 0 issues O += P V in three passes (both operands in shared memory).
// Every hand-off is one mbarrier (commit after each MMA group) and a CTA
// barrier; shared memory written by threads is made visible to the tensor
// cores with fence.proxy.async before the MMAs that read it.  At the end of a
// group the output and L = m + log l are written; after the history group
// the optional fused merge combines both groups by their LSE.
#include "internal.h"

namespace ispa {

namespace {

constexpr int kThreads = 128;
constexpr int kTileQ = 128, kTK = 64;

template <int D>
struct Tf32Cfg {
  static constexpr int kColO = 0, kColS = D, kColQh = D + kTK, kColQl = 2 * D + kTK;
  static constexpr uint32_t kCols = (3 * D + kTK) <= 256 ? 256u : 512u;
  static constexpr int kKBytes = kTK * D * 4;       // K tile: D/32 column blocks of kTK x 128 B
  static constexpr int kVBytes = D * kTK * 4;       // V^T tile: kTK/32 column blocks of D x 128 B
  static constexpr int kPBytes = kTileQ * kTK * 4;  // P tile: kTK/32 column blocks of 128 x 128 B
  static constexpr int kSmem = 2 * (kKBytes + kVBytes + kPBytes) + 1024 + 64;
};

struct Tf32Params {
  int H, Lq, q_tiles;
  int n_ranges, n_loc_ranges;
  int r_begin[3], r_end[3];
  float scale;
  void *o_loc, *o_hist, *o_full;
  float *l_loc, *l_hist, *l_full;
  DevErr err;
};

__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// D[tmem] (+)= A[tmem] * B[smem], kind::tf32
__device__ __forceinline__ void mma_ts_tf32(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Byte offset of element (row, k) of a K-major 128-byte-swizzled fp32 operand
// with `rows` rows: column block k / 32 of rows x 128 bytes; inside it the
// 16-byte chunk (k % 32) / 4 of the row is stored at chunk index XOR (row % 8).
__device__ __forceinline__ uint32_t kmajor_off(int row, int k, int rows) {
  const int blk = k >> 5, kk = k & 31;
  return (uint32_t)(blk * rows * 128 + row * 128 + ((((kk >> 2) ^ (row & 7))) << 4) + ((kk & 3) << 2));
}

// Descriptor of the K step kk (8 elements) of a K-major swizzled operand of `rows` rows.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int kk, int rows) {
  return smem_desc_sw128(base + (uint32_t)((kk >> 2) * rows * 128 + (kk & 3) * 32), 16, 1024);
}

template <typename T>
__device__ __forceinline__ void store_as(T *p, float x);
template <>
__device__ __forceinline__ void store_as<float>(float *p, float x) { *p = x; }
template <>
__device__ __forceinline__ void store_as<__nv_bfloat16>(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

__device__ __forceinline__ void split_tf32(float x, float &hi, float &lo) {
  hi = to_tf32_rn(x);
  lo = to_tf32_rn(x - hi);
}

template <int D, typename TO>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tf32_kernel(const float *__restrict__ q, const float *__restrict__ k, const float *__restrict__ v, int Lkv,
                     Tf32Params P) {
  using Cfg = Tf32Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *k_hi = base, *k_lo = k_hi + Cfg::kKBytes;
  uint8_t *v_hi = k_lo + Cfg::kKBytes, *v_lo = v_hi + Cfg::kVBytes;
  uint8_t *p_hi = v_lo + Cfg::kVBytes, *p_lo = p_hi + Cfg::kPBytes;
  uint64_t *bar = reinterpret_cast<uint64_t *>(p_lo + Cfg::kPBytes);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar + 1);
  int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
  volatile int *abort = abort_flag;

  const int t = threadIdx.x, warp = t >> 5;
  const int slot = blockIdx.x / P.q_tiles;
  const int b = slot / P.H, h = slot % P.H;
  const int qrow = (blockIdx.x % P.q_tiles) * kTileQ + t;
  const bool row_ok = qrow < P.Lq;
  const int H = P.H;
  const long long head_row = ((long long)b * P.Lq + (row_ok ? qrow : 0)) * H + h;

  if (t == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, Cfg::kCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);

  // Q row: hi and lo parts into TMEM (A operand of S = Q K^T)
  {
    const float *qr = q + head_row * D;
#pragma unroll
    for (int c = 0; c < D; c += 16) {
      uint32_t hi[16], lo[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float x = row_ok ? qr[c + i] : 0.f, xh, xl;
        split_tf32(x, xh, xl);
        hi[i] = __float_as_uint(xh);
        lo[i] = __float_as_uint(xl);
      }
      tmem_st16(lane_base + Cfg::kColQh + c, hi);
      tmem_st16(lane_base + Cfg::kColQl + c, lo);
    }
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t idesc_s = make_idesc(128, kTK, 2, 0, 0);  // tf32 A (TMEM) x tf32 B (K-major)
  const uint32_t idesc_pv = make_idesc(128, D, 2, 0, 0);   // tf32 A (K-major) x tf32 B (K-major)
  const uint32_t a_khi = smem_u32(k_hi), a_klo = smem_u32(k_lo), a_vhi = smem_u32(v_hi), a_vlo = smem_u32(v_lo);
  const uint32_t a_phi = smem_u32(p_hi), a_plo = smem_u32(p_lo);
  uint32_t phase = 0;
  bool ok = true;
  const float log2e = 1.4426950408889634f;
  const float sl2 = P.scale * log2e;

  TO *o_loc = reinterpret_cast<TO *>(P.o_loc) + head_row * D;
  TO *o_hist = P.o_hist ? reinterpret_cast<TO *>(P.o_hist) + head_row * D : nullptr;
  TO *o_full = P.o_full ? reinterpret_cast<TO *>(P.o_full) + head_row * D : nullptr;
  float L_loc = -INFINITY;
  const bool has_hist = P.n_ranges > P.n_loc_ranges;

  // groups: 0 = local (ranges [0, n_loc_ranges)), 1 = history
  for (int grp = 0; grp < 2 && ok; ++grp) {
    const int r_first = grp == 0 ? 0 : P.n_loc_ranges, r_last = grp == 0 ? P.n_loc_ranges : P.n_ranges;
    float m = -INFINITY, l = 0.f;  // log2 units
    bool first_pv = true;
    for (int r = r_first; r < r_last && ok; ++r) {
      for (int t0 = P.r_begin[r]; t0 < P.r_end[r] && ok; t0 += kTK) {
        const int n_valid = min(kTK, P.r_end[r] - t0);
        // ---- 1. K and V^T tiles (split) into shared memory
        for (int e = t; e < kTK * D; e += kThreads) {
          const int j = e / D, c = e % D;
          float kx = 0.f, vx = 0.f;
          if (j < n_valid) {
            const long long off = (((long long)b * Lkv + t0 + j) * H + h) * D + c;
            kx = k[off];
            vx = v[off];
          }
          float hi, lo;
          split_tf32(kx, hi, lo);
          *reinterpret_cast<float *>(k_hi + kmajor_off(j, c, kTK)) = hi;
          *reinterpret_cast<float *>(k_lo + kmajor_off(j, c, kTK)) = lo;
          split_tf32(vx, hi, lo);
          *reinterpret_cast<float *>(v_hi + kmajor_off(c, j, D)) = hi;
          *reinterpret_cast<float *>(v_lo + kmajor_off(c, j, D)) = lo;
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        // ---- 2. S = Q K^T, three passes
        if (t == 0) {
          tc_fence_after();
          int n = 0;
#pragma unroll 1
          for (int pass = 0; pass < 3; ++pass) {
            const uint32_t a = tmem + (pass == 2 ? Cfg::kColQl : Cfg::kColQh);
            const uint32_t bb = pass == 1 ? a_klo : a_khi;
#pragma unroll 1
            for (int kk = 0; kk < D / 8; ++kk, ++n)
              mma_ts_tf32(tmem + Cfg::kColS, a + kk * 8, kmajor_desc(bb, kk, kTK), idesc_s, n > 0 ? 1u : 0u);
          }
          mma_commit(bar);
        }
        ok = wait_parity(bar, phase, P.err, abort, 71);
        phase ^= 1;
        if (!__syncthreads_and(ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // ---- 3. softmax of this row; P (hi, lo) into shared memory
        float s[kTK];
        {
          uint32_t raw[32];
#pragma unroll
          for (int c = 0; c < kTK; c += 32) {
            tmem_ld32(lane_base + Cfg::kColS + c, raw);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) s[c + i] = c + i < n_valid ? __uint_as_float(raw[i]) * sl2 : -INFINITY;
          }
        }
        float mt = -INFINITY;
#pragma unroll
        for (int i = 0; i < kTK; ++i) mt = fmaxf(mt, s[i]);
        const float m_new = fmaxf(m, mt);
        const float corr = (m == -INFINITY) ? 0.f : exp2f(m - m_new);
        if (!first_pv && corr != 1.f) {  // O (complete: PV of the previous tile preceded S) scales by corr
#pragma unroll 1
          for (int c = 0; c < D; c += 32) {
            uint32_t o[32];
            tmem_ld32(lane_base + Cfg::kColO + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * corr);
            tmem_st16(lane_base + Cfg::kColO + c, *reinterpret_cast<uint32_t(*)[16]>(&o[0]));
            tmem_st16(lane_base + Cfg::kColO + c + 16, *reinterpret_cast<uint32_t(*)[16]>(&o[16]));
          }
          tmem_wait_st();
        }
        m = m_new;
        float ls = 0.f;
#pragma unroll
        for (int i = 0; i < kTK; ++i) {
          const float p = exp2f(s[i] - m);
          ls += p;
          float hi, lo;
          split_tf32(p, hi, lo);
          *reinterpret_cast<float *>(p_hi + kmajor_off(t, i, kTileQ)) = hi;
          *reinterpret_cast<float *>(p_lo + kmajor_off(t, i, kTileQ)) = lo;
        }
        l = l * corr + ls;
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        // ---- 4. O += P V, three passes
        if (t == 0) {
          tc_fence_after();
          int n = 0;
#pragma unroll 1
          for (int pass = 0; pass < 3; ++pass) {
            const uint32_t pa = pass == 2 ? a_plo : a_phi;
            const uint32_t vb = pass == 1 ? a_vlo : a_vhi;
#pragma unroll 1
            for (int kk = 0; kk < kTK / 8; ++kk, ++n)
              mma_ss(tmem + Cfg::kColO, kmajor_desc(pa, kk, kTileQ), kmajor_desc(vb, kk, D), idesc_pv,
                     (first_pv && n == 0) ? 0u : 1u, 1);
          }
          mma_commit(bar);
        }
        first_pv = false;
        ok = wait_parity(bar, phase, P.err, abort, 72);
        phase ^= 1;
        if (!__syncthreads_and(ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
    }
    if (!ok) break;
    // ---- group end: O / l and L = (m + log2 l) ln 2; the history group merges with the local one
    const bool is_loc = grp == 0;
    const bool empty = first_pv;  // no tile in this group (the local group always has the current chunk)
    const float L = empty ? -INFINITY : (m + log2f(l)) * 0.69314718055994530942f;
    const float inv_l = empty ? 0.f : 1.f / l;
    float wa = 1.f, wb = 0.f, L_full = L;
    if (!is_loc) {
      if (empty) {
        wa = 1.f;
        wb = 0.f;
        L_full = L_loc;
      } else {
        const float mxl = fmaxf(L_loc, L);
        const float ea = expf(L_loc - mxl), eb = expf(L - mxl), se = ea + eb;
        wa = ea / se;
        wb = eb / se;
        L_full = mxl + logf(se);
      }
    }
    if (row_ok) {
      if (is_loc) {
        L_loc = L;
        P.l_loc[head_row] = L;
      } else if (P.l_hist) {
        P.l_hist[head_row] = L;
      }
    }
    TO *dst = is_loc ? o_loc : o_hist;
    const bool write_full = o_full != nullptr && !is_loc;
#pragma unroll 1
    for (int c = 0; c < D; c += 32) {
      float xo[32];
      if (!empty) {
        uint32_t raw[32];
        tmem_ld32(lane_base + Cfg::kColO + c, raw);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) xo[i] = __uint_as_float(raw[i]) * inv_l;
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) xo[i] = 0.f;
      }
      if (!row_ok) continue;
      if (dst) {
#pragma unroll
        for (int i = 0; i < 32; ++i) store_as(dst + c + i, xo[i]);
      }
      if (write_full) {
#pragma unroll
        for (int i = 0; i < 32; ++i) store_as(o_full + c + i, wa * load_as_float(o_loc + c + i) + wb * xo[i]);
      }
    }
    if (write_full && row_ok) P.l_full[head_row] = L_full;
    tc_fence_before();
    __syncthreads();  // O is read before the next group's first PV overwrites it
    tc_fence_after();
    if (!has_hist) {  // the history group is empty: O_hist = 0, L_hist = -inf, O_full = O_loc
      if (row_ok) {
        if (o_hist)
          for (int c = 0; c < D; ++c) store_as(o_hist + c, 0.f);
        if (P.l_hist) P.l_hist[head_row] = -INFINITY;
        if (o_full) {
          for (int c = 0; c < D; ++c) store_as(o_full + c, load_as_float(o_loc + c));
          P.l_full[head_row] = L_loc;
        }
      }
      break;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, Cfg::kCols);
}

template <int D, typename TO>
ispa_status launch_tf32_typed(const float *q, const float *k, const float *v, int B, int Lkv, const Tf32Params &P,
                              cudaStream_t s) {
  using Cfg = Tf32Cfg<D>;
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e =
        cudaFuncSetAttribute(attn_tf32_kernel<D, TO>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem);
    if (e != cudaSuccess) return cuda_status(e, "tf32 attention smem attribute");
    configured_device = dev;
  }
  attn_tf32_kernel<D, TO><<<dim3(B * P.H * P.q_tiles), kThreads, Cfg::kSmem, s>>>(q, k, v, Lkv, P);
  note_launch();
  return cuda_status(cudaGetLastError(), "tf32 attention launch");
}

}  // namespace

ispa_status launch_attn_tf32(const ispa_attn_desc &d, const GroupRanges &g, float scale, const float *q,
                             const float *k, const float *v, void *o_loc, float *l_loc, void *o_hist, float *l_hist,
                             void *o_full, float *l_full, cudaStream_t s) {
  if (g.Lq == 0) return ISPA_OK;
  Tf32Params P{};
  ispa_status st = device_err(&P.err);
  if (st != ISPA_OK) return st;
  P.H = d.H;
  P.Lq = g.Lq;
  P.q_tiles = (g.Lq + kTileQ - 1) / kTileQ;
  for (int r = 0; r < g.n_loc; ++r) {
    P.r_begin[P.n_ranges] = g.loc_begin[r];
    P.r_end[P.n_ranges] = g.loc_end[r];
    ++P.n_ranges;
  }
  P.n_loc_ranges = P.n_ranges;
  if (g.hist_end > g.hist_begin) {
    P.r_begin[P.n_ranges] = g.hist_begin;
    P.r_end[P.n_ranges] = g.hist_end;
    ++P.n_ranges;
  }
  P.scale = scale;
  P.o_loc = o_loc;
  P.o_hist = o_hist;
  P.o_full = o_full;
  P.l_loc = l_loc;
  P.l_hist = l_hist;
  P.l_full = l_full;
  const bool bf = d.out_dtype == ISPA_BF16;
  switch (d.head_dim) {
    case 32:
      return bf ? launch_tf32_typed<32, __nv_bfloat16>(q, k, v, d.B, g.Lkv, P, s)
                : launch_tf32_typed<32, float>(q, k, v, d.B, g.Lkv, P, s);
    case 64:
      return bf ? launch_tf32_typed<64, __nv_bfloat16>(q, k, v, d.B, g.Lkv, P, s)
                : launch_tf32_typed<64, float>(q, k, v, d.B, g.Lkv, P, s);
    default:
      return bf ? launch_tf32_typed<128, __nv_bfloat16>(q, k, v, d.B, g.Lkv, P, s)
                : launch_tf32_typed<128, float>(q, k, v, d.B, g.Lkv, P, s);
  }
}

}  // namespace ispa
