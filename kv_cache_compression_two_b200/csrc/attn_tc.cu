// attn_tc.cu -- two-group attention on tcgen05 tensor cores (bf16 in, fp32 accumulate, d = 128).
//
// One CTA computes one 128-query tile of one head of one instance and walks the
// KV tiles of the local group (sink range, then current range) followed by the
// history group.  Each group keeps its own online-softmax state; at the end of
// a group the normalised output and its log-sum-exp are written, and after the
// history group the optional fused merge combines both groups by their LSE.
//
// Warp roles (256 threads, one CTA per SM):
//   warps 0, 2  TMA producers of the K and of the V tiles (128 keys x 128
//               dims), each through a three-stage ring with full/empty barriers.
//   warp 1      TMEM allocator and MMA issuer.  S_j = Q K_j^T (bf16; Q from
//               tensor memory, K from shared memory) into S buffer j % 2, and
//               PV_j: O += P_j V_j (fp16 P from tensor memory, fp16 V from shared
//               memory).  Order: S_0, S_1, then per tile j: PV_j, S_{j+2}, issued
//               back to back once P_j is published (the copies of V_j and
//               K_{j+2} are waited for before P_j).
//   warp 3      idle.
//   warps 4-7   Q into tensor memory once; then per tile the softmax (one row
//               per thread, TMEM lane = row), the correction of O when the
//               running maximum grows, and the group epilogues.
//
// TMEM columns: O [0,128), S buffers [128,256) and [256,384), Q [384,448)
// (bf16 pairs).  P_j is written as packed fp16 into the first 64 columns of
// the buffer that held S_j.  Because S is double-buffered, S_{j+1} is already
// computed while the softmax works on S_j, so the softmax runs back to back
// and the tensor pipe works on PV_j and S_{j+2} meanwhile.
//
// Ordering argument (tcgen05.mma operations issued by one thread execute in
// order, and a commit fires once all earlier operations have completed):
//   * S_{j+2} reuses the buffer of S_j / P_j: it is issued after PV_j (which
//     reads P_j) and after P_j was published, i.e. after the softmax finished
//     reading S_j.
//   * When the softmax of tile j starts (S_j complete), PV_{j-2} has completed
//     (S_j was issued after it); PV_{j-1} may still run, so a correction of O
//     first waits for PV_{j-1}; PV_j itself waits for P_j.  PV_j commits to
//     o_done[j % 2], so a wait names its PV by index and the barrier it waits
//     on cannot be a phase ahead (its next PV, PV_{j+2}, needs P_{j+2}) nor
//     behind in a way the parity would hide.
//   * At the end of the local group the epilogue reads O after PV of that tile
//     (o_done) and releases it (o_free) before the first history PV, which
//     starts O afresh, is issued.
#include <algorithm>

#include "internal.h"

namespace ispa {

namespace {

constexpr int kThreads = 256;  // warps 0-3: K producer, MMA issuer, V producer, idle; warps 4-7: softmax
constexpr int kTileQ = 128, kTileK = 128, kD = 128;
constexpr int kBoxBytes = 128 * 128;          // 128 rows x 64 bf16
constexpr int kTileBytes = 2 * kBoxBytes;     // 128 rows x 128 bf16
constexpr int kStagesK = 3, kStagesV = 3;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS = 128, kColQ = 384;  // S buffer b at kColS + 128 b
constexpr float kRescaleThreshold = 8.0f;     // log2 units

struct AttnParams {
  int H, Lq;
  int q_tiles;             // 128-query tiles per (instance, head); CTA x: slot x / q_tiles, tile x % q_tiles
  int n_ranges;            // ranges 0..n_ranges-1; the first n_loc_ranges are local
  int n_loc_ranges;
  int r_begin[3], r_end[3];
  int n_loc_tiles, n_tiles;
  float scale_log2;        // softmax scale * log2(e)
  const float *v_unscale;  // [B * H]: 2^-s of the fp16 copy of V (see prepare_v)
  void *o_loc, *o_hist, *o_full;
  float *l_loc, *l_hist, *l_full;
  // Statistics operands (fp32 outputs only; see launch_attn_tc): when set, the
  // epilogue writes dA = tf32(O_full - O_loc) here, and leaves tf32(O_loc) in
  // o_loc, the operands of the absorption statistics.
  float *stats_dA;
  DevErr err;
};

// ---------------------------------------------------------------------------
// fp16 copy of V.  P = exp(S - m) is rounded to 16 bits before the PV product;
// in fp16 (11 significant bits) that rounding is 8x finer than in bf16, which
// keeps the output error well inside the parity tolerance.  tcgen05 kind::f16
// needs both operands in the same type, so V is converted once per call.  A
// bf16 value (8 significant bits) is exact in fp16 when its magnitude lies in
// [2^-17, 65504], and below 2^-14 fp16 keeps an absolute spacing of 2^-24, so
// a converted entry is off by at most 2^-25.  One pass converts V as it is and
// records, per head of each instance, the largest |v| and the sum of v^2.  A
// head whose largest |v| reaches 2^15 (overflow margin), or whose RMS is
// below 2^-10 (where 2^-25 would no longer be small against the 2^-11
// relative rounding of its typical entries), is converted again by a second
// kernel with a power-of-two scale 2^s that puts its largest |v| in
// [2^14, 2^15), and the epilogue multiplies O by 2^-s (exact); for the other
// heads that kernel only writes 2^-s = 1.  Only the rows the tiles read are
// converted: every range rounded up to whole 128-row tiles.
// ---------------------------------------------------------------------------
struct VPrep {
  int B, H, Lkv;
  int n_ext;
  int ext_begin[3], ext_end[3];  // row extents the tiles touch
};

// Conversion pass.  Each thread keeps one 16-byte column group c8 (8 values
// of one head) and walks rows, converting them unscaled; the 16 lanes that
// cover one head combine their largest |v| and sum of squares by shuffles and
// one lane per head issues the atomics (non-negative floats order like their
// bit patterns).
__global__ void __launch_bounds__(256) v_prep_kernel(VPrep p, const __nv_bfloat16 *__restrict__ v, __half *v16,
                                                     unsigned int *amax_bits, float *sumsq) {
  const int D = p.H * kD;
  const int vec_per_row = D / 8;                       // multiple of 16 (kD / 8 = 16 per head)
  const int b = blockIdx.y;
  const int lanes = gridDim.x * blockDim.x;
  const int row_step = lanes / vec_per_row;            // rows advanced per pass (>= 1 by the launch)
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  const int c8 = tid % vec_per_row;
  const int r0 = tid / vec_per_row;
  float mx = 0.f, ss = 0.f;
  if (r0 < row_step) {
    for (int e = 0; e < p.n_ext; ++e)
      for (int row = p.ext_begin[e] + r0; row < p.ext_end[e]; row += row_step) {
        const long long off = ((long long)b * p.Lkv + row) * D + c8 * 8;
        const uint4 in = __ldg(reinterpret_cast<const uint4 *>(v + off));
        const uint32_t w[4] = {in.x, in.y, in.z, in.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[j]));
          mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
          ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
          __half2 hh = __floats2half2_rn(f.x, f.y);
          o[j] = *reinterpret_cast<uint32_t *>(&hh);
        }
        *reinterpret_cast<uint4 *>(v16 + off) = make_uint4(o[0], o[1], o[2], o[3]);
      }
  }
  // vec_per_row = 16 H and warps start at multiples of 32, so lanes 16k..16k+15
  // hold the 16 column groups of one head of one row: reduce them by shuffles.
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
  }
  if ((threadIdx.x & 15) == 0 && r0 < row_step) {
    atomicMax(amax_bits + b * p.H + (c8 * 8) / kD, __float_as_uint(mx));
    atomicAdd(sumsq + b * p.H + (c8 * 8) / kD, ss);
  }
}

__device__ __forceinline__ int v_exponent(unsigned int amax_bits) {
  const float a = __uint_as_float(amax_bits);
  if (!(a > 0.f) || !isfinite(a)) return 0;
  return 14 - ilogbf(a);  // a * 2^s in [2^14, 2^15)
}

// The heads the unscaled copy does not serve (see the note above): largest
// |v| from 2^15 up, or RMS below 2^-10 (sum of squares below count * 2^-20).
__device__ __forceinline__ bool v_needs_scale(unsigned int amax_bits, float sumsq, float count) {
  return !(__uint_as_float(amax_bits) < 32768.f) || sumsq < count * 0x1p-20f;
}

// Second pass: v_unscale for every head, and the scaled copy of the heads
// v_needs_scale picks (same thread layout as v_prep_kernel).
__global__ void __launch_bounds__(256) v_fix_kernel(VPrep p, const __nv_bfloat16 *__restrict__ v, __half *v16,
                                                    const unsigned int *__restrict__ amax_bits,
                                                    const float *__restrict__ sumsq, float *v_unscale) {
  const int D = p.H * kD;
  const int vec_per_row = D / 8;
  const int b = blockIdx.y;
  const int lanes = gridDim.x * blockDim.x;
  const int row_step = lanes / vec_per_row;
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  const int c8 = tid % vec_per_row;
  const int r0 = tid / vec_per_row;
  if (r0 >= row_step) return;
  const int hb = b * p.H + (c8 * 8) / kD;
  float count = 0.f;
  for (int e = 0; e < p.n_ext; ++e) count += (float)(p.ext_end[e] - p.ext_begin[e]) * kD;
  const bool fix = v_needs_scale(amax_bits[hb], sumsq[hb], count);
  const int sexp = fix ? v_exponent(amax_bits[hb]) : 0;
  if (r0 == 0 && (c8 * 8) % kD == 0) v_unscale[hb] = ldexpf(1.f, -sexp);
  if (!fix) return;
  const float scale = ldexpf(1.f, sexp);
  for (int e = 0; e < p.n_ext; ++e)
    for (int row = p.ext_begin[e] + r0; row < p.ext_end[e]; row += row_step) {
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

// ---------------------------------------------------------------------------
// Prepared fp16 copy of V (ispa_v16_prepare): the same conversion, kept by the
// caller across calls so that each call converts only the frames it writes.
// Per (instance, head) the copy holds v * 2^e with one exponent e; its state
// records e, 2^-e, the largest |v| and the sum of v^2 over the rows prepared so
// far (and their count), by which the rule above picks e.  A prepare converts
// its rows with the current e; when the new rows move a head's e, every row of
// that head is converted again from v with the new one.
// ---------------------------------------------------------------------------
struct V16State {
  float *unscale;      // 2^-e
  int *expo;           // e
  unsigned int *amax;  // largest |v| (bits of a non-negative float)
  float *sumsq;        // sum of v^2
  double *count;       // values accumulated
  int *flag;           // 1: e changed in the last prepare, the head is converted again
};

__host__ __device__ inline size_t v16_a256(size_t x) { return (x + 255) & ~size_t(255); }

V16State v16_state(void *v16, int B, int H, int Lkv) {
  char *base = static_cast<char *>(v16) + v16_a256((size_t)B * Lkv * H * kD * 2);
  const size_t w = v16_a256((size_t)B * H * 4);
  V16State st;
  st.unscale = reinterpret_cast<float *>(base);
  st.expo = reinterpret_cast<int *>(base + w);
  st.amax = reinterpret_cast<unsigned int *>(base + 2 * w);
  st.sumsq = reinterpret_cast<float *>(base + 3 * w);
  st.count = reinterpret_cast<double *>(base + 4 * w);
  st.flag = reinterpret_cast<int *>(base + 4 * w + v16_a256((size_t)B * H * 8));
  return st;
}

// Conversion of the prepared rows (thread layout of v_prep_kernel), scaled by
// each head's current 2^e; the statistics are taken on the unscaled values.
__global__ void __launch_bounds__(256) v16_prep_kernel(VPrep p, const __nv_bfloat16 *__restrict__ v, __half *v16,
                                                       V16State st) {
  const int D = p.H * kD;
  const int vec_per_row = D / 8;
  const int b = blockIdx.y;
  const int lanes = gridDim.x * blockDim.x;
  const int row_step = lanes / vec_per_row;
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  const int c8 = tid % vec_per_row;
  const int r0 = tid / vec_per_row;
  const int hb = b * p.H + (c8 * 8) / kD;
  const float scale = r0 < row_step ? ldexpf(1.f, st.expo[hb]) : 1.f;
  float mx = 0.f, ss = 0.f;
  if (r0 < row_step) {
    for (int e = 0; e < p.n_ext; ++e)
      for (int row = p.ext_begin[e] + r0; row < p.ext_end[e]; row += row_step) {
        const long long off = ((long long)b * p.Lkv + row) * D + c8 * 8;
        const uint4 in = __ldg(reinterpret_cast<const uint4 *>(v + off));
        const uint32_t w[4] = {in.x, in.y, in.z, in.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[j]));
          mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
          ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
          const float lo = fminf(fmaxf(f.x * scale, -65504.f), 65504.f);
          const float hi = fminf(fmaxf(f.y * scale, -65504.f), 65504.f);
          __half2 hh = __floats2half2_rn(lo, hi);
          o[j] = *reinterpret_cast<uint32_t *>(&hh);
        }
        *reinterpret_cast<uint4 *>(v16 + off) = make_uint4(o[0], o[1], o[2], o[3]);
      }
  }
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
  }
  if ((threadIdx.x & 15) == 0 && r0 < row_step) {
    atomicMax(st.amax + hb, __float_as_uint(mx));
    atomicAdd(st.sumsq + hb, ss);
  }
}

// One thread per (instance, head): the exponent the rule picks for the rows
// prepared so far; a change marks the head for conversion again.
__global__ void __launch_bounds__(256) v16_decide_kernel(int BH, double added, V16State st) {
  for (int hb = blockIdx.x * blockDim.x + threadIdx.x; hb < BH; hb += gridDim.x * blockDim.x) {
    const double count = st.count[hb] + added;
    st.count[hb] = count;
    const int e = v_needs_scale(st.amax[hb], st.sumsq[hb], (float)count) ? v_exponent(st.amax[hb]) : 0;
    st.flag[hb] = e != st.expo[hb] ? 1 : 0;
    st.expo[hb] = e;
    st.unscale[hb] = ldexpf(1.f, -e);
  }
}

// Every row [0, Lkv) of the heads whose exponent changed, converted again.
__global__ void __launch_bounds__(256) v16_reconvert_kernel(VPrep p, const __nv_bfloat16 *__restrict__ v, __half *v16,
                                                            V16State st) {
  const int D = p.H * kD;
  const int vec_per_row = D / 8;
  const int b = blockIdx.y;
  const int lanes = gridDim.x * blockDim.x;
  const int row_step = lanes / vec_per_row;
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  const int c8 = tid % vec_per_row;
  const int r0 = tid / vec_per_row;
  if (r0 >= row_step) return;
  const int hb = b * p.H + (c8 * 8) / kD;
  if (!st.flag[hb]) return;
  const float scale = ldexpf(1.f, st.expo[hb]);
  for (int row = r0; row < p.Lkv; row += row_step) {
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

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

struct SmemLayout {
  uint8_t k[kStagesK][kTileBytes];
  uint8_t v[kStagesV][kTileBytes];
  uint64_t k_full[kStagesK], k_empty[kStagesK];
  uint64_t v_full[kStagesV], v_empty[kStagesV];
  uint64_t q_ready;   // Q is in tensor memory (128 arrivals)
  uint64_t s_full[2]; // S_j complete in buffer j % 2
  uint64_t p_full[2]; // P_j written into buffer j % 2 (128 arrivals)
  uint64_t o_done[2]; // PV_j complete, on o_done[j % 2]
  uint64_t o_free;    // the local-group epilogue has read O (128 arrivals)
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int rng[8];  // range begins [0,3), ends [3,6), count [6]: read by the tile walks
};

constexpr int kSmemBytes = sizeof(SmemLayout) + 1024;

// Walks the tile sequence: local ranges first, then history.
// The ranges come from shared memory (copied from the parameters at the start):
// an indexed load of a kernel parameter sat on the softmax's per-tile path.
struct TileIter {
  int range, t0;
  __device__ void start(const int *rng) {
    range = 0;
    t0 = rng[6] > 0 ? rng[0] : 0;
  }
  __device__ int valid(const int *rng) const { return min(kTileK, rng[3 + range] - t0); }
  __device__ void next(const int *rng) {
    t0 += kTileK;
    if (t0 >= rng[3 + range]) {
      ++range;
      if (range < rng[6]) t0 = rng[range];
    }
  }
};

// max(a, b, c) in one instruction (sm_100); a NaN operand is ignored as by fmaxf.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

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
    attn_tc_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                   const __nv_bfloat16 *__restrict__ q, AttnParams P) {
  extern __shared__ uint8_t smem_raw[];
  SmemLayout &sm =
      *reinterpret_cast<SmemLayout *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  volatile int *abort = &sm.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slot = blockIdx.x / P.q_tiles;  // (instance, head) = b * H + h
  const int b = slot / P.H, h = slot % P.H;
  const int q0 = (blockIdx.x % P.q_tiles) * kTileQ;
  const bool has_hist = P.n_tiles > P.n_loc_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesK; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
    }
    for (int s = 0; s < kStagesV; ++s) {
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    mbar_init(&sm.q_ready, 128);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.p_full[s], 128);
    }
    mbar_init(&sm.o_done[0], 1);
    mbar_init(&sm.o_done[1], 1);
    mbar_init(&sm.o_free, 128);
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    for (int r = 0; r < 3; ++r) {
      sm.rng[r] = P.r_begin[r];
      sm.rng[3 + r] = P.r_end[r];
    }
    sm.rng[6] = P.n_ranges;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
  }
  if (warp == 1) tmem_alloc(&sm.tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0 || warp == 2) {
    // ------------------------------------------------------------ producers: K (warp 0), V (warp 2)
    if (lane == 0) {
      const bool is_k = warp == 0;
      const int n_stages = is_k ? kStagesK : kStagesV;
      const CUtensorMap *map = is_k ? &tk : &tv;
      uint64_t *full = is_k ? sm.k_full : sm.v_full;
      uint64_t *empty = is_k ? sm.k_empty : sm.v_empty;
      const int x0 = h * kD;
      uint32_t pend = 0, ph_bits = 0;
      TileIter it;
      it.start(sm.rng);
      for (int j = 0; j < P.n_tiles; ++j, it.next(sm.rng)) {
        const int st = j % n_stages;
        const uint32_t ph = (j / n_stages) & 1;
        if (!wait_parity(&empty[st], ph ^ 1, P.err, abort, is_k ? 11 : 12)) break;
        uint8_t *dst = is_k ? sm.k[st] : sm.v[st];
        mbar_arrive_expect_tx(&full[st], kTileBytes);
        tma_load_4d(dst, map, &full[st], 0, it.t0, x0 / 64, b);  // both 64-column halves, one box
        pend |= 1u << st;
        ph_bits = (ph_bits & ~(1u << st)) | (ph << st);
      }
      if (*abort) {  // let copies in flight land before the CTA exits
        for (int st = 0; st < n_stages; ++st)
          if (pend & (1u << st)) wait_parity_drain(&full[st], (ph_bits >> st) & 1, P.err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = make_idesc(128, 128, 1, 0, 0);  // bf16 Q (TMEM) x bf16 K (K-major)
      const uint32_t idesc_pv = make_idesc(128, 128, 0, 0, 1);  // fp16 P (TMEM) x fp16 V (MN-major)
      // Descriptors of every ring stage, built once: each MMA then costs the
      // issuing thread (which shares its scheduler with a softmax warp) only an
      // add.  The start-address field (bits 0-13, address / 16) does not carry
      // out for shared-memory offsets below 256 KiB.
      uint64_t dk[kStagesK], dv[kStagesV];
#pragma unroll
      for (int st = 0; st < kStagesK; ++st) dk[st] = smem_desc_sw128(smem_u32(sm.k[st]), 16, 1024);
#pragma unroll
      for (int st = 0; st < kStagesV; ++st) dv[st] = smem_desc_sw128(smem_u32(sm.v[st]), kBoxBytes, 1024);
      auto pick = [](const uint64_t *d, int n, int st) {  // register-resident select of d[st]
        uint64_t r = d[0];
#pragma unroll
        for (int i = 1; i < n; ++i) r = st == i ? d[i] : r;
        return r;
      };
      auto issue_s = [&](int j) {  // S_j = Q K_j^T into buffer j & 1
        const uint64_t kd = pick(dk, kStagesK, j % kStagesK);
        const uint32_t d_s = tmem + kColS + (uint32_t)(j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk)
          mma_ts(d_s, tmem + kColQ + (uint32_t)kk * 8, kd + (uint64_t)(((kk >> 2) * kBoxBytes + (kk & 3) * 32) >> 4),
                 idesc_qk, kk > 0 ? 1u : 0u);
        mma_commit(&sm.s_full[j & 1]);
        mma_commit(&sm.k_empty[j % kStagesK]);
      };
      auto issue_pv = [&](int j) {  // O (+)= P_j V_j, P_j in the first 64 columns of buffer j & 1
        const bool first = (j == 0) || (j == P.n_loc_tiles);
        const uint64_t vd = pick(dv, kStagesV, j % kStagesV);
        const uint32_t a_p = tmem + kColS + (uint32_t)(j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < kTileK / 16; ++kk)
          mma_ts(tmem + kColO, a_p + kk * 8, vd + (uint64_t)((kk * 2048) >> 4), idesc_pv,
                 (first && kk == 0) ? 0u : 1u);
        mma_commit(&sm.o_done[j & 1]);
        mma_commit(&sm.v_empty[j % kStagesV]);
      };
      bool ok = wait_parity(&sm.q_ready, 0, P.err, abort, 20);
      for (int j = 0; ok && j < 2 && j < P.n_tiles; ++j) {
        ok = wait_parity(&sm.k_full[j % kStagesK], (j / kStagesK) & 1, P.err, abort, 21);
        if (!ok) break;
        tc_fence_after();
        issue_s(j);
      }
      for (int j = 0; ok && j < P.n_tiles; ++j) {
        const int jn = j + 2;  // S runs two tiles ahead, into the buffer PV_j reads
        // The copies of V_j and K_{j+2} are waited for first: they land long
        // before the softmax of tile j ends, so these waits overlap the MMAs
        // still queued, and the only wait between P_j and the 16 MMAs of PV_j
        // and S_{j+2} is P_j itself.  (No cycle: the stages of V_j and K_{j+2}
        // were released by PV_{j-3} and S_{j-1}, issued earlier.)
        ok = wait_parity(&sm.v_full[j % kStagesV], (j / kStagesV) & 1, P.err, abort, 25);
        if (ok && jn < P.n_tiles)
          ok = wait_parity(&sm.k_full[jn % kStagesK], (jn / kStagesK) & 1, P.err, abort, 26);
        if (ok) ok = wait_parity_spin(&sm.p_full[j & 1], (uint32_t)(j >> 1) & 1, P.err, abort, 23);
        if (ok && j == P.n_loc_tiles) ok = wait_parity(&sm.o_free, 0, P.err, abort, 24);
        if (!ok) break;
        tc_fence_after();
        issue_pv(j);
        if (jn < P.n_tiles) issue_s(jn);
      }
      if (!ok) {
        mma_commit(&sm.drain);
        wait_parity_drain(&sm.drain, 0, P.err);
      }
    }
  } else if (warp >= 4) {
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
    // This row of Q into TMEM as the A operand of S = Q K^T: column c holds
    // elements 2c and 2c + 1 (zeros past the end of the sequence).
    {
      const uint4 *src = reinterpret_cast<const uint4 *>(q + head_row * kD);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t w[16];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint4 v = row_ok ? __ldg(src + c * 4 + u) : make_uint4(0u, 0u, 0u, 0u);
          w[4 * u] = v.x;
          w[4 * u + 1] = v.y;
          w[4 * u + 2] = v.z;
          w[4 * u + 3] = v.w;
        }
        tmem_st16(lane_base + kColQ + c * 16, w);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.q_ready);
    }
    float m_ref = 0.f, l = 0.f, L_loc = -INFINITY;
    TileIter it;
    it.start(sm.rng);
    for (int j = 0; j < P.n_tiles; ++j, it.next(sm.rng)) {
      const bool grp_first = (j == 0) || (j == P.n_loc_tiles);
      const bool grp_last = (j == P.n_loc_tiles - 1) || (j == P.n_tiles - 1);
      const int n_valid = it.valid(sm.rng);
      const uint32_t col_s = kColS + (uint32_t)(j & 1) * 128;
      bool ok = wait_parity_spin(&sm.s_full[j & 1], (uint32_t)(j >> 1) & 1, P.err, abort, 31);
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
      // row maximum with three-input max instructions: 64 for 128 values, in
      // eight independent chains
      float mx[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) mx[t] = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; c += 2)
        mx[(c >> 1) & 7] = fmax3(mx[(c >> 1) & 7], __uint_as_float(sr[c >> 5][c & 31]),
                                 __uint_as_float(sr[(c + 1) >> 5][(c + 1) & 31]));
      const float mt = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) *
                       P.scale_log2;
      if (grp_first) {
        m_ref = mt;
        l = 0.f;
      } else if (__any_sync(0xffffffffu, mt > m_ref + kRescaleThreshold)) {
        // O may still be accumulating PV_{j-1}; it is final once that PV lands (PV_j
        // waits for P_j, which this warpgroup has not published yet).
        ok = wait_parity(&sm.o_done[(j - 1) & 1], (uint32_t)((j - 1) >> 1) & 1, P.err, abort, 32);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after();
        const float m_new = fmaxf(m_ref, mt);
        const float f = ex2(m_ref - m_new);
        m_ref = m_new;
        l *= f;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(lane_base + kColO + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * f);
          tmem_st16(lane_base + kColO + c * 32, *reinterpret_cast<uint32_t(*)[16]>(&o[0]));
          tmem_st16(lane_base + kColO + c * 32 + 16, *reinterpret_cast<uint32_t(*)[16]>(&o[16]));
        }
      }
      // P = exp2(s * scale * log2e - m_ref) <= 2^8, packed to fp16 pairs into columns [0, 64) of the buffer.
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
      mbar_arrive(&sm.p_full[j & 1]);

      if (!grp_last) continue;
      // ---- end of a group: O is final once PV_j has landed (PV_{j+1} needs P_{j+1},
      // which this warpgroup has not produced, so the wait cannot alias).
      ok = wait_parity(&sm.o_done[j & 1], (uint32_t)(j >> 1) & 1, P.err, abort, 33);
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
        tmem_ld32(lane_base + kColO + c * 32, raw);
        tmem_wait_ld();
        float xo[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) xo[t] = __uint_as_float(raw[t]) * inv_l;
        if (!row_ok) continue;
        if (dst) store_row32<TO>(dst + c * 32, xo);
        if (write_full) {
          float y[32];
          if (!is_loc) {
            load_row32<TO>(o_loc + c * 32, y);
#pragma unroll
            for (int t = 0; t < 32; ++t) xo[t] = wa * y[t] + wb * xo[t];
          } else {
#pragma unroll
            for (int t = 0; t < 32; ++t) y[t] = xo[t];  // no history: O_full = O_loc
          }
          store_row32<TO>(o_full + c * 32, xo);
          if (P.stats_dA) {  // the statistics operands, rounded as the statistics pass rounds them
            float da[32];
#pragma unroll
            for (int t = 0; t < 32; ++t) {
              da[t] = to_tf32_rn(xo[t] - y[t]);
              y[t] = to_tf32_rn(y[t]);
            }
            store_row32<float>(P.stats_dA + head_row * kD + c * 32, da);
            store_row32<TO>(o_loc + c * 32, y);
          }
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
ispa_status launch_typed(const CUtensorMap &tk, const CUtensorMap &tv, const __nv_bfloat16 *q, const AttnParams &P,
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
  dim3 grid(B * P.H * P.q_tiles);
  attn_tc_kernel<TO><<<grid, kThreads, kSmemBytes, s>>>(tk, tv, q, P);
  note_launch();
  return cuda_status(cudaGetLastError(), "tcgen05 attention launch");
}

// K or V [B, rows, D] (16-bit, D = H * 128) seen as (64 columns of a 128-byte
// block, row, block of the row, instance): the block stride (128 bytes) is
// below the row stride, so that one box {64, 128, 2, 1} brings both 64-column
// halves of a head's 128-row tile, half after half as the swizzled operand
// layout wants them (half the copy instructions of two 16 KB boxes; the
// launch time is the same either way, the copies not being the bound here).
ispa_status map_kv16(CUtensorMap *m, const void *base, int D, int rows, int B, CUtensorMapDataType dt) {
  const uint64_t dims[4] = {64, (uint64_t)rows, (uint64_t)D / 64, (uint64_t)B};
  const uint64_t strides[3] = {(uint64_t)D * 2, 128, (uint64_t)D * 2 * (uint64_t)rows};
  const uint32_t box[4] = {64, 128, 2, 1};
  return make_tmap(m, dt, 4, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

size_t attn_tc_workspace_bytes(int B, int H, int Lkv, int v_layout) {
  if (v_layout == ISPA_V_F16_PREPARED) return 0;
  if (v_layout == ISPA_KV_E4M3_PREPARED) return attn_f8_workspace_bytes(B, H);
  return a256((size_t)B * Lkv * H * kD * 2) + 3 * a256((size_t)B * H * 4);
}

size_t v16_state_offset(int B, int H, int Lkv) { return a256((size_t)B * Lkv * H * kD * 2); }

size_t v16_state_bytes(int B, int H) { return 4 * a256((size_t)B * H * 4) + a256((size_t)B * H * 8) + a256((size_t)B * H * 4); }

size_t v16_bytes(int B, int H, int Lkv) { return v16_state_offset(B, H, Lkv) + v16_state_bytes(B, H); }

ispa_status launch_v16_prepare(int B, int H, int Lkv, int row_begin, int row_end, const void *v, void *v16,
                               cudaStream_t s) {
  const int D = H * kD;
  V16State st = v16_state(v16, B, H, Lkv);
  cudaError_t e = cudaSuccess;
  if (row_begin == 0) {  // a prepare from the first frame starts the copy afresh
    e = cudaMemsetAsync(static_cast<char *>(v16) + v16_state_offset(B, H, Lkv), 0, v16_state_bytes(B, H), s);
    if (e != cudaSuccess) return cuda_status(e, "prepared V state clear");
  }
  VPrep vp{};
  vp.B = B;
  vp.H = H;
  vp.Lkv = Lkv;
  vp.n_ext = 1;
  vp.ext_begin[0] = row_begin;
  vp.ext_end[0] = row_end;
  const int vec_per_row = D / 8;
  const __nv_bfloat16 *vb = static_cast<const __nv_bfloat16 *>(v);
  __half *out = static_cast<__half *>(v16);
  if (row_end > row_begin) {
    const int rows = row_end - row_begin;
    const int want = std::max(1, (int)(((long long)rows * vec_per_row + 255) / 256));
    const int blocks = std::max((vec_per_row + 255) / 256, std::min(want, (sm_count() * 8 + B - 1) / B));
    v16_prep_kernel<<<dim3(blocks, B), 256, 0, s>>>(vp, vb, out, st);
    note_launch();
  }
  const int BH = B * H;
  v16_decide_kernel<<<(BH + 255) / 256, 256, 0, s>>>(BH, (double)(row_end - row_begin) * kD, st);
  const int fix_blocks = std::max((vec_per_row + 255) / 256, 2);
  v16_reconvert_kernel<<<dim3(fix_blocks, B), 256, 0, s>>>(vp, vb, out, st);
  note_launch(2);
  return cuda_status(cudaGetLastError(), "prepared V launch");
}

ispa_status launch_prepared(const ispa_attn_desc &d, const GroupRanges &g, float scale, const void *q,
                            const CUtensorMap &tk, const CUtensorMap &tv, AttnParams &P, void *o_loc, float *l_loc,
                            void *o_hist, float *l_hist, void *o_full, float *l_full, cudaStream_t s,
                            float *stats_dA);

ispa_status launch_attn_tc(const ispa_attn_desc &d, const GroupRanges &g, float scale, const void *q,
                           const void *k, const void *v, void *o_loc, float *l_loc, void *o_hist, float *l_hist,
                           void *o_full, float *l_full, void *workspace, cudaStream_t s, float *stats_dA) {
  if (g.Lq == 0) return ISPA_OK;
  if (d.v_layout == ISPA_KV_E4M3_PREPARED)  // k is the prepared fp8 K/V, v is not used
    return launch_attn_f8(d, g, scale, q, k, o_loc, l_loc, o_hist, l_hist, o_full, l_full, workspace, s);
  AttnParams P{};
  ispa_status st = device_err(&P.err);
  if (st != ISPA_OK) return st;
  const int D = d.H * kD;

  CUtensorMap tk, tv;
  if ((st = map_kv16(&tk, k, D, g.Lkv, d.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16)) != ISPA_OK) return st;
  if (d.v_layout == ISPA_V_F16_PREPARED) {
    // the caller's prepared copy (ispa_v16_prepare) and its per-head 2^-e
    P.v_unscale = v16_state(const_cast<void *>(v), d.B, d.H, g.Lkv).unscale;
    if ((st = map_kv16(&tv, v, D, g.Lkv, d.B, CU_TENSOR_MAP_DATA_TYPE_FLOAT16)) != ISPA_OK) return st;
    return launch_prepared(d, g, scale, q, tk, tv, P, o_loc, l_loc, o_hist, l_hist, o_full, l_full, s, stats_dA);
  }
  // ---- fp16 copy of the V rows the tiles read (workspace)
  char *ws = static_cast<char *>(workspace);
  __half *v16 = reinterpret_cast<__half *>(ws);
  const size_t head_words = a256((size_t)d.B * d.H * 4);
  unsigned int *amax = reinterpret_cast<unsigned int *>(ws + a256((size_t)d.B * g.Lkv * D * 2));
  float *sumsq = reinterpret_cast<float *>(reinterpret_cast<char *>(amax) + head_words);
  float *v_unscale = reinterpret_cast<float *>(reinterpret_cast<char *>(amax) + 2 * head_words);
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
  cudaError_t e = cudaMemsetAsync(amax, 0, 2 * head_words, s);  // amax and sumsq
  if (e != cudaSuccess) return cuda_status(e, "attention workspace clear");
  const int vec_per_row = D / 8;
  const int prep_blocks = max((vec_per_row + 255) / 256, (sm_count() * 8 + d.B - 1) / d.B);
  const int fix_blocks = max((vec_per_row + 255) / 256, 2);
  const __nv_bfloat16 *vb = static_cast<const __nv_bfloat16 *>(v);
  v_prep_kernel<<<dim3(prep_blocks, d.B), 256, 0, s>>>(vp, vb, v16, amax, sumsq);
  v_fix_kernel<<<dim3(fix_blocks, d.B), 256, 0, s>>>(vp, vb, v16, amax, sumsq, v_unscale);
  note_launch(2);
  if ((st = cuda_status(cudaGetLastError(), "V conversion launch")) != ISPA_OK) return st;
  P.v_unscale = v_unscale;
  if ((st = map_kv16(&tv, v16, D, g.Lkv, d.B, CU_TENSOR_MAP_DATA_TYPE_FLOAT16)) != ISPA_OK) return st;
  return launch_prepared(d, g, scale, q, tk, tv, P, o_loc, l_loc, o_hist, l_hist, o_full, l_full, s, stats_dA);
}

// The attention launch proper, once V is in fp16 (tv) with its unscale in P.
ispa_status launch_prepared(const ispa_attn_desc &d, const GroupRanges &g, float scale, const void *q,
                            const CUtensorMap &tk, const CUtensorMap &tv, AttnParams &P, void *o_loc, float *l_loc,
                            void *o_hist, float *l_hist, void *o_full, float *l_full, cudaStream_t s,
                            float *stats_dA) {
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
  P.stats_dA = (d.out_dtype == ISPA_F32 && o_full) ? stats_dA : nullptr;
  P.l_loc = l_loc;
  P.l_hist = l_hist;
  P.l_full = l_full;
  const __nv_bfloat16 *qb = static_cast<const __nv_bfloat16 *>(q);
  if (d.out_dtype == ISPA_F32) return launch_typed<float>(tk, tv, qb, P, d.B, s);
  return launch_typed<__nv_bfloat16>(tk, tv, qb, P, d.B, s);
}

}  // namespace ispa
