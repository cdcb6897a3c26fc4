// attn_tc.cu -- two-group attention on tcgen05 tensor cores (bf16 in, fp32 accumulate, d = 128).
//
// One CTA computes two 128-query tiles (A and B, 256 queries) of one head of
// one instance and walks the KV tiles of the local group (sink range, then
// current range) followed by the history group.  Both query tiles share every
// K/V tile, which halves the operand traffic from L2 per FLOP -- the limit of a
// single-tile design on this part.  Each group keeps its own online-softmax
// state; at the end of a group the normalised output and its log-sum-exp are
// written, and after the history group the optional fused merge combines both
// groups by their LSE.
//
// Warp roles (384 threads, one CTA per SM; setmaxnreg moves registers from the
// control warpgroup, 64 per thread, to the softmax warpgroups, 216 per thread):
//   warp 0      TMA producer: Q_A and Q_B once, then K and V tiles (128 keys x
//               128 dims) through two-stage rings with separate K and V barriers.
//   warp 1      TMEM allocator and MMA issuer, per KV tile j:
//                 PV_{j-1}(A), S_j(A), PV_{j-1}(B), S_j(B)
//               with S_j(X) = Q_X K_j^T (bf16, operands in shared memory) and
//               PV_j(X): O_X += P_j(X) V_j (fp16 P read from TMEM as operand A,
//               fp16 V from shared memory), so the softmax of one query tile
//               overlaps the MMAs of the other.
//   warps 2-3   idle (they complete the control warpgroup).
//   warps 4-7   softmax / correction / epilogue of query tile A, one row per
//   warps 8-11  thread (TMEM lane = row); the same for query tile B.
//
// TMEM columns: S_A [0,128) S_B [128,256) O_A [256,384) O_B [384,512).  P_j(X)
// is written as packed fp16 into columns [0,64) of S_X after the softmax has
// read S_j(X); tcgen05.mma operations issued by one thread execute in order,
// so PV_j(X) has read P before S_{j+1}(X) overwrites the columns.
//
// Ordering argument:
//   * S_{j+1}(X) is issued after the softmax published P_j(X), i.e. after it
//     finished its tcgen05.ld of S_j(X).
//   * S_j(X) is issued after PV_{j-1}(X); its commit (s_full) therefore also
//     covers PV_{j-1}(X), so while the softmax of tile j runs no MMA touches
//     O_X and it may rescale O_X directly; PV_j(X) waits for P_j(X).
//   * At the end of the local group the epilogue reads O_X after PV of that
//     tile (o_done) and releases it (o_free) before the first history PV
//     overwrites it.
#include <functional>
#include <map>
#include <mutex>
#include <queue>
#include <tuple>
#include <vector>

#include "internal.h"

namespace ispa {

namespace {

constexpr int kThreads = 384;  // control warpgroup (producer, MMA, 2 idle) + one softmax warpgroup per query tile
constexpr int kRegsControl = 64, kRegsSoftmax = 216;
constexpr int kMinLaunchRegs = (128 * kRegsControl + 256 * kRegsSoftmax + kThreads - 1) / kThreads;
constexpr int kTileQ = 128, kTileK = 128, kD = 128;
constexpr int kBoxBytes = 128 * 128;          // 128 rows x 64 bf16
constexpr int kTileBytes = 2 * kBoxBytes;     // 128 rows x 128 bf16
constexpr int kStagesK = 3, kStagesV = 2;  // K is needed one MMA step earlier than V
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;  // + 128 * query tile
constexpr float kRescaleThreshold = 8.0f;     // log2 units

struct AttnParams {
  int H, Lq;
  // Work items over the B * H (instance, head) slots g = b * H + h, each with
  // q_tiles 128-query tiles: first the CTAs with two tiles -- pair_base + 1
  // pairs for slots g < pair_extra, pair_base for the others -- then the CTAs
  // with one tile for the rest (see choose_pairs).
  int q_tiles, pair_base, pair_extra, n_pair_items;
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
  uint8_t q[2][kTileBytes];
  uint8_t k[kStagesK][kTileBytes];
  uint8_t v[kStagesV][kTileBytes];
  uint64_t q_full;
  uint64_t k_full[kStagesK], k_empty[kStagesK];
  uint64_t v_full[kStagesV], v_empty[kStagesV];
  uint64_t s_full[2], p_full[2], o_done[2], o_free[2];  // per query tile
  uint64_t drain;
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

// Packed fp32 pair arithmetic (sm_100): one instruction for two lanes of work.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
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
  // work item: (instance, head, first query tile, one or two tiles)
  int nx = 2, b, h, q0;
  {
    const int pe = P.pair_extra, pb = P.pair_base;
    int item = blockIdx.x, g, k;
    if (item < P.n_pair_items) {
      if (item < pe * (pb + 1)) {
        g = item / (pb + 1);
        k = item % (pb + 1);
      } else {
        item -= pe * (pb + 1);
        g = pe + item / pb;
        k = item % pb;
      }
      q0 = 2 * k * kTileQ;
    } else {
      nx = 1;
      item -= P.n_pair_items;
      const int s_hi = P.q_tiles - 2 * (pb + 1), s_lo = P.q_tiles - 2 * pb;  // singles per slot
      if (item < pe * s_hi) {
        g = item / s_hi;
        k = 2 * (pb + 1) + item % s_hi;
      } else {
        item -= pe * s_hi;
        g = pe + item / s_lo;
        k = 2 * pb + item % s_lo;
      }
      q0 = k * kTileQ;
    }
    b = g / P.H;
    h = g % P.H;
  }
  const bool has_hist = P.n_tiles > P.n_loc_tiles;

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kStagesK; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
    }
    for (int s = 0; s < kStagesV; ++s) {
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sm.s_full[x], 1);
      mbar_init(&sm.p_full[x], 128);
      mbar_init(&sm.o_done[x], 1);
      mbar_init(&sm.o_free[x], 128);
    }
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

  // Register split: the control warpgroup (warps 0-3: producer, MMA issuer, two
  // idle warps) gives registers to the two softmax warpgroups.  The block is
  // launched with 384 x 168; 128 x kRegsControl + 256 x kRegsSoftmax must not
  // exceed that (the launcher checks the compiled count before launching).
  // Each role sits inside the branch that set its register budget, so the
  // compiler allocates every role against its own limit.
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const int x0 = h * kD;
      mbar_arrive_expect_tx(&sm.q_full, nx * kTileBytes);
      for (int x = 0; x < nx; ++x) {
        tma_load_3d(sm.q[x], &tq, &sm.q_full, x0, q0 + x * kTileQ, b);
        tma_load_3d(sm.q[x] + kBoxBytes, &tq, &sm.q_full, x0 + 64, q0 + x * kTileQ, b);
      }
      uint32_t k_pend = 0, v_pend = 0, k_ph = 0, v_ph = 0;
      TileIter it;
      it.start(P);
      for (int j = 0; j < P.n_tiles; ++j, it.next(P)) {
        const int sk = j % kStagesK, sv = j % kStagesV;
        const uint32_t phk = (j / kStagesK) & 1, phv = (j / kStagesV) & 1;
        if (!wait_parity(&sm.k_empty[sk], phk ^ 1, P.err, abort, 11)) break;
        mbar_arrive_expect_tx(&sm.k_full[sk], kTileBytes);
        tma_load_3d(sm.k[sk], &tk, &sm.k_full[sk], x0, it.t0, b);
        tma_load_3d(sm.k[sk] + kBoxBytes, &tk, &sm.k_full[sk], x0 + 64, it.t0, b);
        k_pend |= 1u << sk;
        k_ph = (k_ph & ~(1u << sk)) | (phk << sk);
        if (!wait_parity(&sm.v_empty[sv], phv ^ 1, P.err, abort, 12)) break;
        mbar_arrive_expect_tx(&sm.v_full[sv], kTileBytes);
        tma_load_3d(sm.v[sv], &tv, &sm.v_full[sv], x0, it.t0, b);
        tma_load_3d(sm.v[sv] + kBoxBytes, &tv, &sm.v_full[sv], x0 + 64, it.t0, b);
        v_pend |= 1u << sv;
        v_ph = (v_ph & ~(1u << sv)) | (phv << sv);
      }
      if (*abort) {  // let copies in flight land before the CTA exits
        wait_parity_drain(&sm.q_full, 0, P.err);
        for (int s = 0; s < kStagesK; ++s)
          if (k_pend & (1u << s)) wait_parity_drain(&sm.k_full[s], (k_ph >> s) & 1, P.err);
        for (int s = 0; s < kStagesV; ++s)
          if (v_pend & (1u << s)) wait_parity_drain(&sm.v_full[s], (v_ph >> s) & 1, P.err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = make_idesc(128, 128, 1, 0, 0);  // bf16 Q x bf16 K, both K-major
      const uint32_t idesc_pv = make_idesc(128, 128, 0, 0, 1);  // fp16 P (TMEM) x fp16 V (MN-major)
      auto issue_s = [&](int j, int x) {  // S_j(x) = Q_x K_j^T
        const uint32_t q_addr = smem_u32(sm.q[x]);
        const uint32_t k_addr = smem_u32(sm.k[j % kStagesK]);
        const uint32_t d_s = tmem + kColS + (uint32_t)x * 128;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (uint32_t)(kk >> 2) * kBoxBytes + (uint32_t)(kk & 3) * 32;
          mma_ss(d_s, smem_desc_sw128(q_addr + off, 16, 1024), smem_desc_sw128(k_addr + off, 16, 1024), idesc_qk,
                 kk > 0 ? 1u : 0u, 0);
        }
        mma_commit(&sm.s_full[x]);
      };
      auto issue_pv = [&](int j, int x) {  // O_x (+)= P_j(x) V_j, P in the first 64 columns of S_x
        const bool first = (j == 0) || (j == P.n_loc_tiles);
        const uint32_t v_addr = smem_u32(sm.v[j % kStagesV]);
        const uint32_t a_p = tmem + kColS + (uint32_t)x * 128;
#pragma unroll
        for (int kk = 0; kk < kTileK / 16; ++kk)
          mma_ts(tmem + kColO + (uint32_t)x * 128, a_p + kk * 8,
                 smem_desc_sw128(v_addr + kk * 2048, kBoxBytes, 1024), idesc_pv, (first && kk == 0) ? 0u : 1u);
        mma_commit(&sm.o_done[x]);
      };
      bool ok = wait_parity(&sm.q_full, 0, P.err, abort, 21) &&
                wait_parity(&sm.k_full[0], 0, P.err, abort, 22);
      if (ok) {
        tc_fence_after();
        for (int x = 0; x < nx; ++x) issue_s(0, x);
        mma_commit(&sm.k_empty[0]);
      }
      for (int j = 0; ok && j < P.n_tiles; ++j) {
        const int sv = j % kStagesV;
        const bool more = j + 1 < P.n_tiles;
        const int sk1 = (j + 1) % kStagesK;
        for (int x = 0; x < nx && ok; ++x) {
          ok = wait_parity_spin(&sm.p_full[x], (uint32_t)(j & 1), P.err, abort, 23);
          if (ok && j == P.n_loc_tiles) ok = wait_parity(&sm.o_free[x], 0, P.err, abort, 24);
          if (ok && x == 0) ok = wait_parity(&sm.v_full[sv], (j / kStagesV) & 1, P.err, abort, 25);
          if (!ok) break;
          tc_fence_after();
          issue_pv(j, x);
          if (x == nx - 1) mma_commit(&sm.v_empty[sv]);
          if (more) {
            // K_{j+1} is waited for only after PV_j(x) is queued
            if (x == 0) ok = wait_parity(&sm.k_full[sk1], ((j + 1) / kStagesK) & 1, P.err, abort, 26);
            if (!ok) break;
            tc_fence_after();
            issue_s(j + 1, x);
            if (x == nx - 1) mma_commit(&sm.k_empty[sk1]);
          }
        }
      }
      if (!ok) {
        mma_commit(&sm.drain);
        wait_parity_drain(&sm.drain, 0, P.err);
      }
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    // ------------------------------------------------------------ softmax + epilogue
    const int x = (warp - 4) >> 2;  // query tile of this warpgroup
    if (x < nx) {
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // row inside the tile == TMEM lane
    const int qrow = q0 + x * kTileQ + r;
    const bool row_ok = qrow < P.Lq;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t col_s = kColS + (uint32_t)x * 128, col_o = kColO + (uint32_t)x * 128;
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
      bool ok = wait_parity_spin(&sm.s_full[x], (uint32_t)(j & 1), P.err, abort, 31);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      uint32_t sr[4][32];  // S row of this thread (fp32 bits), straight from TMEM
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(lane_base + col_s + c * 32, sr[c]);
      tmem_wait_ld();
      if (n_valid < kTileK) {  // ragged tile: keys past the range end get -inf
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= n_valid) sr[c >> 5][c & 31] = 0xff800000u;
      }
      float mx[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) mx[t] = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) mx[c & 7] = fmaxf(mx[c & 7], __uint_as_float(sr[c >> 5][c & 31]));
      const float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                             fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) *
                       P.scale_log2;
      if (grp_first) {
        m_ref = mt;
        l = 0.f;
      } else if (__any_sync(0xffffffffu, mt > m_ref + kRescaleThreshold)) {
        // O_x is quiescent here (PV_{j-1}(x) completed before S_j(x)); PV_j(x) waits for P_j(x).
        const float m_new = fmaxf(m_ref, mt);
        const float f = ex2(m_ref - m_new);
        m_ref = m_new;
        l *= f;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(lane_base + col_o + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * f);
          tmem_st16(lane_base + col_o + c * 32, *reinterpret_cast<uint32_t(*)[16]>(&o[0]));
          tmem_st16(lane_base + col_o + c * 32 + 16, *reinterpret_cast<uint32_t(*)[16]>(&o[16]));
        }
      }
      // P = exp2(s * scale * log2e - m_ref) <= 2^8, packed to fp16 pairs into columns [0, 64) of S_x.
      const float2 sc2 = make_float2(P.scale_log2, P.scale_log2), nm2 = make_float2(-m_ref, -m_ref);
      float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const float2 x = ffma2(make_float2(__uint_as_float(sr[c][2 * t]), __uint_as_float(sr[c][2 * t + 1])), sc2, nm2);
          const float2 pp = make_float2(ex2(x.x), ex2(x.y));
          ls[t & 1] = fadd2(ls[t & 1], pp);
          pk[t] = pack_f16x2(pp.x, pp.y);
        }
        tmem_st16(lane_base + col_s + c * 16, pk);
      }
      tmem_wait_st();
      l += (ls[0].x + ls[0].y) + (ls[1].x + ls[1].y);
      tc_fence_before();
      mbar_arrive(&sm.p_full[x]);

      if (!grp_last) continue;
      // ---- end of a group: O_x is final once PV_j(x) has landed (o_done counts the
      // PVs of this tile; PV_{j-1}(x) completed before S_j(x), so the wait is exact).
      ok = wait_parity(&sm.o_done[x], (uint32_t)(j & 1), P.err, abort, 33);
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
        const float mxl = fmaxf(L_loc, L);
        const float ea = expf(L_loc - mxl), eb = expf(L - mxl), se = ea + eb;
        wa = ea / se;
        wb = eb / se;
        L_full = mxl + logf(se);
      }
      TO *dst = is_loc ? o_loc : o_hist;
      const bool write_full = o_full != nullptr && (!is_loc || !has_hist);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t raw[32];
        tmem_ld32(lane_base + col_o + c * 32, raw);
        tmem_wait_ld();
        float xo[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) xo[t] = __uint_as_float(raw[t]) * inv_l;
        if (!row_ok) continue;
        if (dst) store_row32<TO>(dst + c * 32, xo);
        if (write_full) {
          if (!is_loc) {
            float y[32];
            load_row32<TO>(o_loc + c * 32, y);
#pragma unroll
            for (int t = 0; t < 32; ++t) xo[t] = wa * y[t] + wb * xo[t];
          }
          store_row32<TO>(o_full + c * 32, xo);
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
        mbar_arrive(&sm.o_free[x]);
      }
    }
    }  // x < nx
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// Splits the T query tiles of each of the `slots` (instance, head) pairs into
// CTAs of two tiles (best use of each K/V tile) and of one tile.  The two-tile
// CTAs are numbered first and the hardware dispatches CTAs roughly in order,
// so the one-tile CTAs fill the last wave.  The number of two-tile CTAs is
// chosen by simulating that greedy dispatch on n_sm SMs with a one-tile CTA
// costing kSingleCost of a two-tile one; results are cached per shape.
void choose_pairs(int T, int slots, int n_sm, int *pair_base, int *pair_extra) {
  constexpr double kSingleCost = 0.67;  // measured ratio of one-tile to two-tile CTA time
  static std::mutex mu;
  static std::map<std::tuple<int, int, int>, std::pair<int, int>> cache;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_tuple(T, slots, n_sm);
  auto hit = cache.find(key);
  if (hit == cache.end()) {
    const long long max_pairs = (long long)slots * (T / 2);
    const long long tiles = (long long)slots * T;
    double best = 1e300;
    long long best_n = max_pairs;
    for (long long n = max_pairs; n >= 0; --n) {
      std::priority_queue<double, std::vector<double>, std::greater<double>> q;
      for (int i = 0; i < n_sm; ++i) q.push(0.0);
      double end = 0.0;
      const long long n_single = tiles - 2 * n;
      for (long long i = 0; i < n + n_single; ++i) {
        const double t1 = q.top() + (i < n ? 1.0 : kSingleCost);
        q.pop();
        end = t1 > end ? t1 : end;
        q.push(t1);
      }
      if (end < best - 1e-9) {
        best = end;
        best_n = n;
      }
      if (n + n_sm < best_n) break;  // far fewer pairs than the best only adds singles
    }
    hit = cache.emplace(key, std::make_pair((int)(best_n / slots), (int)(best_n % slots))).first;
  }
  *pair_base = hit->second.first;
  *pair_extra = hit->second.second;
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
    // setmaxnreg.inc waits for registers the block does not have if the launch
    // allocation is smaller than the split; refuse to launch in that case.
    cudaFuncAttributes fa[2];
    e = cudaFuncGetAttributes(&fa[0], attn_tc_kernel<float>);
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa[1], attn_tc_kernel<__nv_bfloat16>);
    if (e != cudaSuccess) return cuda_status(e, "attention attributes");
    if (fa[0].numRegs < kMinLaunchRegs || fa[1].numRegs < kMinLaunchRegs)
      return fail(ISPA_ERR_CUDA, "attention kernel compiled with %d/%d registers, the register split needs %d",
                  fa[0].numRegs, fa[1].numRegs, kMinLaunchRegs);
    configured_device = dev;
  }
  dim3 grid(B * P.H * P.q_tiles - P.n_pair_items);  // every pair CTA stands for two tiles
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
  choose_pairs(P.q_tiles, d.B * d.H, sm_count(), &P.pair_base, &P.pair_extra);
  P.n_pair_items = d.B * d.H * P.pair_base + P.pair_extra;
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
