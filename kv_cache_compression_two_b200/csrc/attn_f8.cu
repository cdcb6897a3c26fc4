// attn_f8.cu -- two-group attention with fp8 e4m3 products (tcgen05 kind::f8f6f4), d = 128.
//
// The post-switch layers combined with 8-bit quantisation [EN-notes, Key
// Findings (Figure 7); DE-summary 4, "Beschleunigung"]: Q, K and V in e4m3 with
// one fp32 scale per (instance, head), S = Q K^T and O = P V on the 8-bit
// tensor cores with fp32 accumulation, P in e4m3.  The scheme:
//   * s_X = amax_X / 448 over the head's rows, codes e4m3(x * (448 / amax_X));
//   * t = S s_q s_k scale log2(e); per group and query row a reference m: the
//     first 128-key tile's maximum, moved to a later tile's maximum only when
//     that exceeds m by more than 2.75 (O and the sum then scaled by
//     2^(m_old - m_new)); p = 2^(t - m + 6) <= 2^8.75 < 448 (finite in e4m3,
//     the weights of the bulk of the keys in its normal range), l += p in
//     fp32, O += e4m3(p) V8;
//   * O = O s_v / l, L = (m - 6 + log2 l) ln 2, the groups merged by their LSE.
// The softmax forms a tile's weights against the current reference and finds
// the tile's maximum in the same pass; only when the maximum passes the
// threshold (after the first tiles of a group, rarely) does it wait for the
// previous PV, rescale O and form the weights again.
// The tiles of a key range start at its first key rounded down to a multiple
// of 16 (the 16-byte rule of the transposed V copy's TMA coordinate); keys of
// a tile outside the range are masked.
//
// K and V come prepared (ispa_kv8_prepare): K8 [B, Lkv, H, 128] bytes and V8
// transposed, [B, H, 128, Lkv_pad] bytes, so that both products read their B
// operand K-major; the per-head scales sit in the prepared buffer's state.  Q
// is quantised on its way into tensor memory, with the per-head amax that a
// pre-pass of the call finds.
//
// Warp roles (256 threads, one CTA per SM), as in the bf16 kernel:
//   warps 0, 2  TMA producers of the K8 and of the V8 tiles (16 KB each), four
//               stages each.
//   warp 1      TMEM allocator and MMA issuer: S_j = Q8 K8_j^T into S buffer
//               j % 2 (4 MMAs of K = 32), PV_j: O += P8_j V8_j (4 MMAs).
//   warps 4-7   Q8 into tensor memory; per tile the softmax (one row per
//               thread), the correction of O, the group epilogues.
// TMEM columns: O [0,128), S [128,256) and [256,384), Q8 [384,416) (four e4m3
// per column), P8 [416,448) and [448,480).  P has buffers of its own, so the
// S buffer of tile j is free as soon as the softmax has read it: S_{j+2} is
// issued then (barrier s_free), not after PV_j as in the bf16 kernel where P
// overwrites S -- the tensor pipe always holds the next S while the softmax
// works, and only PV_j waits for P_j.
//
// Ordering argument (tcgen05.mma operations of one thread run in order; a
// commit fires when all earlier ones have completed):
//   * S_{j+2} overwrites S buffer j % 2 after s_free(j): the softmax of tile j
//     has finished its tcgen05.ld of S_j.
//   * P_j goes to P buffer j % 2 once PV_{j-2} (pv_done) has read P_{j-2}.
//   * PV_j commits to pv_done[j % 2], so each barrier advances once per two
//     PVs and a wait names its PV by index: the correction of O in the softmax
//     of tile j waits for PV_{j-1} (PVs complete in order, so PV_{j-2} too) --
//     with S issued ahead of PV, PV_{j-2} may still be running when S_j has
//     landed, and one barrier over every PV would then be two phases behind;
//     the next phase of pv_done[(j-1) % 2] is PV_{j+1}, which waits for
//     P_{j+1}, so the wait cannot alias.  The same barriers free P buffers.
//   * At the end of the local group the epilogue reads O after PV of that tile
//     and releases it (o_free) before the first history PV starts O afresh.
//   * s_free and p_full count one arrival per softmax warp: lane 0 arrives
//     after the warp's tcgen05.wait (the load, or the store, of all 32 lanes
//     has completed), a tcgen05 fence and a __syncwarp.
#include <algorithm>

#include <cuda_fp8.h>

#include "internal.h"

namespace ispa {

namespace {

constexpr int kThreads = 256;
constexpr int kTileQ = 128, kTileK = 128, kD = 128;
constexpr int kTileBytes = 128 * 128;  // 128 rows x 128 bytes
constexpr int kStagesK = 4, kStagesV = 4;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS = 128, kColQ = 384, kColP = 416;
constexpr float kPOffset = 6.0f;  // p = 2^(t - m + 6)
constexpr float kTau = 2.75f;     // m moves when a tile's maximum exceeds it by more: p <= 2^8.75 < 448
constexpr int kAlign = 16;        // tiles of a range start at a multiple of 16 keys

size_t a256(size_t x) { return (x + 255) & ~size_t(255); }
int pad16(int n) { return (n + 15) / 16 * 16; }

// ---------------------------------------------------------------------------
// prepared buffer: K8, V8 transposed, then the state
// ---------------------------------------------------------------------------
struct KV8State {
  float *scale_k, *scale_v;        // amax / 448
  unsigned int *amax_k, *amax_v;   // largest |x| of the rows prepared (bits of a non-negative float)
  unsigned int *cand_k, *cand_v;   // largest |x| of this prepare's rows
  int *flag;                       // bit 0: K of the head converted again, bit 1: V
};

struct KV8Layout {
  size_t k_off, v_off, st_off, bytes;
  int Lkv_pad;
};

KV8Layout kv8_layout(int B, int H, int Lkv) {
  KV8Layout L;
  L.Lkv_pad = pad16(Lkv);
  L.k_off = 0;
  L.v_off = a256((size_t)B * Lkv * H * kD);
  L.st_off = L.v_off + a256((size_t)B * H * kD * L.Lkv_pad);
  L.bytes = L.st_off + 7 * a256((size_t)B * H * 4);
  return L;
}

KV8State kv8_state(void *base, const KV8Layout &L, int B, int H) {
  char *s = static_cast<char *>(base) + L.st_off;
  const size_t w = a256((size_t)B * H * 4);
  KV8State st;
  st.scale_k = reinterpret_cast<float *>(s);
  st.scale_v = reinterpret_cast<float *>(s + w);
  st.amax_k = reinterpret_cast<unsigned int *>(s + 2 * w);
  st.amax_v = reinterpret_cast<unsigned int *>(s + 3 * w);
  st.cand_k = reinterpret_cast<unsigned int *>(s + 4 * w);
  st.cand_v = reinterpret_cast<unsigned int *>(s + 5 * w);
  st.flag = reinterpret_cast<int *>(s + 6 * w);
  return st;
}

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return (lo & 0xffffu) | (hi << 16);
}

// inv = 448 / amax in fp32 (0 for an all-zero head), the scale amax / 448
__device__ __forceinline__ float q8_inv(float amax) { return amax > 0.f ? 448.f / amax : 0.f; }

// Largest |x| of rows [r0, r1) of a bf16 [B, rows, H, 128] tensor per (instance, head):
// one thread per 16-byte column group, lanes of one head reduced by shuffles.
__global__ void __launch_bounds__(256) amax_rows_kernel(int H, int rows_total, int r0, int r1,
                                                        const __nv_bfloat16 *__restrict__ x, unsigned int *amax) {
  const int D = H * kD, vec_per_row = D / 8, b = blockIdx.y;
  const int row_step = (gridDim.x * blockDim.x) / vec_per_row;
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  const int c8 = tid % vec_per_row, rr = tid / vec_per_row;
  float mx = 0.f;
  if (rr < row_step)
    for (int row = r0 + rr; row < r1; row += row_step) {
      const uint4 in = __ldg(reinterpret_cast<const uint4 *>(x + ((long long)b * rows_total + row) * D + c8 * 8));
      const uint32_t w[4] = {in.x, in.y, in.z, in.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[j]));
        mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 15) == 0 && rr < row_step) atomicMax(amax + b * H + (c8 * 8) / kD, __float_as_uint(mx));
}

// Per head: the running amax grows to cover this prepare's rows; a grown amax
// changes the scale, and the head's rows are converted again (flag).  A reset
// (prepare from row 0) takes this prepare's amax as it is.
__global__ void kv8_decide_kernel(int BH, int reset, KV8State st) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < BH; i += gridDim.x * blockDim.x) {
    int flag = 0;
    const unsigned int ck = st.cand_k[i], cv = st.cand_v[i];
    if (reset) {
      st.amax_k[i] = ck;
      st.amax_v[i] = cv;
    } else {
      if (ck > st.amax_k[i]) { st.amax_k[i] = ck; flag |= 1; }
      if (cv > st.amax_v[i]) { st.amax_v[i] = cv; flag |= 2; }
    }
    st.flag[i] = flag;
    st.scale_k[i] = __uint_as_float(st.amax_k[i]) / 448.f;
    st.scale_v[i] = __uint_as_float(st.amax_v[i]) / 448.f;
    st.cand_k[i] = 0u;
    st.cand_v[i] = 0u;
  }
}

// K rows [r0, r1) -> K8 (same layout, one byte per value); with only_flagged,
// only the heads whose K scale changed.  One thread per 16 values.
__global__ void __launch_bounds__(256) k8_convert_kernel(int H, int Lkv, int r0, int r1, int only_flagged,
                                                         const __nv_bfloat16 *__restrict__ k, uint8_t *k8,
                                                         KV8State st) {
  const int D = H * kD, vec_per_row = D / 16, b = blockIdx.y;
  const int row_step = (gridDim.x * blockDim.x) / vec_per_row;
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  const int c16 = tid % vec_per_row, rr = tid / vec_per_row;
  if (rr >= row_step) return;
  const int hb = b * H + (c16 * 16) / kD;
  if (only_flagged && !(st.flag[hb] & 1)) return;
  const float inv = q8_inv(__uint_as_float(st.amax_k[hb]));
  for (int row = r0 + rr; row < r1; row += row_step) {
    const long long off = ((long long)b * Lkv + row) * D + c16 * 16;
    const uint4 a = __ldg(reinterpret_cast<const uint4 *>(k + off));
    const uint4 c = __ldg(reinterpret_cast<const uint4 *>(k + off + 8));
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[2 * j]));
      const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[2 * j + 1]));
      o[j] = e4m3x4(f0.x * inv, f0.y * inv, f1.x * inv, f1.y * inv);
    }
    *reinterpret_cast<uint4 *>(k8 + off) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// V rows [r0, r1) -> V8 transposed: block (chunk of 64 rows, head, instance)
// reads 64 x 128 values, converts them and writes each of the 128 columns'
// 64 bytes contiguously (keys along the row of the transposed copy).
__global__ void __launch_bounds__(256) v8t_convert_kernel(int H, int Lkv, int Lkv_pad, int r0, int r1,
                                                          int only_flagged, const __nv_bfloat16 *__restrict__ v,
                                                          uint8_t *v8t, KV8State st) {
  __shared__ uint8_t t[kD][64 + 4];
  const int h = blockIdx.y, b = blockIdx.z, hb = b * H + h;
  if (only_flagged && !(st.flag[hb] & 2)) return;
  const int row0 = r0 + blockIdx.x * 64;
  if (row0 >= r1) return;
  const float inv = q8_inv(__uint_as_float(st.amax_v[hb]));
  const int D = H * kD;
  // load: 64 rows x 16 groups of 8 values; 256 threads, 4 passes
  for (int e = threadIdx.x; e < 64 * 16; e += blockDim.x) {
    const int r = e / 16, g = e % 16, row = row0 + r;
    uint32_t packed[2] = {0u, 0u};
    if (row < r1) {
      const uint4 in = __ldg(reinterpret_cast<const uint4 *>(v + ((long long)b * Lkv + row) * D + h * kD + g * 8));
      const uint32_t w[4] = {in.x, in.y, in.z, in.w};
      float f[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 p = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[j]));
        f[2 * j] = p.x * inv;
        f[2 * j + 1] = p.y * inv;
      }
      packed[0] = e4m3x4(f[0], f[1], f[2], f[3]);
      packed[1] = e4m3x4(f[4], f[5], f[6], f[7]);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) t[g * 8 + j][r] = (uint8_t)(packed[j / 4] >> (8 * (j % 4)));
  }
  __syncthreads();
  // store: 128 columns x 64 keys; 16 threads per column write 4 bytes each
  const int nk = min(64, r1 - row0);
  for (int e = threadIdx.x; e < kD * 16; e += blockDim.x) {
    const int col = e / 16, q4 = e % 16;
    uint8_t *dst = v8t + ((long long)hb * kD + col) * Lkv_pad + row0 + q4 * 4;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (q4 * 4 + j < nk) dst[j] = t[col][q4 * 4 + j];
  }
}

// ---------------------------------------------------------------------------
// the attention kernel
// ---------------------------------------------------------------------------
struct AttnParams8 {
  int H, Lq;
  int q_tiles;
  int n_ranges, n_loc_ranges;
  int r_begin[3], r_end[3];
  int n_loc_tiles, n_tiles;
  float scale_log2;
  const unsigned int *q_amax;  // [B * H]
  const float *scale_k, *scale_v;
  void *o_loc, *o_hist, *o_full;
  float *l_loc, *l_hist, *l_full;
  DevErr err;
};

struct SmemLayout8 {
  uint8_t k[kStagesK][kTileBytes];
  uint8_t v[kStagesV][kTileBytes];
  uint64_t k_full[kStagesK], k_empty[kStagesK];
  uint64_t v_full[kStagesV], v_empty[kStagesV];
  uint64_t q_ready;
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2], pv_done[2];  // pv_done[b]: PV_j done for j % 2 == b (P buffer b free again)
  uint64_t o_free, drain;
  uint32_t tmem_base;
  int abort;
  int rng[8];  // range begins [0,3), ends [3,6), count [6]: read by the tile walks
};

constexpr int kSmemBytes8 = sizeof(SmemLayout8) + 1024;

// Tile walk over the ranges: each range's tiles start at its first key rounded
// down to a multiple of 16; lo / hi are the tile's valid columns.
struct TileIter8 {  // the ranges come from shared memory (copied from the parameters at the start)
  int range, t0;
  __device__ void start(const int *rng) {
    range = 0;
    t0 = rng[6] > 0 ? rng[0] - rng[0] % kAlign : 0;
  }
  __device__ int lo(const int *rng) const { return max(0, rng[range] - t0); }
  __device__ int hi(const int *rng) const { return min(kTileK, rng[3 + range] - t0); }
  __device__ void next(const int *rng) {
    t0 += kTileK;
    if (t0 >= rng[3 + range]) {
      ++range;
      if (range < rng[6]) t0 = rng[range] - rng[range] % kAlign;
    }
  }
};

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed fp32 pair arithmetic (sm_100): one instruction for two lanes of work.
__device__ __forceinline__ float2 ffma2f(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

__device__ __forceinline__ float2 fadd2f(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

__device__ __forceinline__ float fmax3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// D[tmem] (+)= A[tmem] * B[smem], kind::f8f6f4 (A is M x 32 bytes of e4m3: 8 columns)
__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

template <typename TO>
__device__ __forceinline__ void store_row32_8(TO *dst, const float (&x)[32]);
template <>
__device__ __forceinline__ void store_row32_8<float>(float *dst, const float (&x)[32]) {
  float4 *d4 = reinterpret_cast<float4 *>(dst);
#pragma unroll
  for (int v = 0; v < 8; ++v) d4[v] = make_float4(x[4 * v], x[4 * v + 1], x[4 * v + 2], x[4 * v + 3]);
}
template <>
__device__ __forceinline__ void store_row32_8<__nv_bfloat16>(__nv_bfloat16 *dst, const float (&x)[32]) {
  uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
  for (int v = 0; v < 4; ++v)
    d4[v] = make_uint4(pack_bf16x2(x[8 * v], x[8 * v + 1]), pack_bf16x2(x[8 * v + 2], x[8 * v + 3]),
                       pack_bf16x2(x[8 * v + 4], x[8 * v + 5]), pack_bf16x2(x[8 * v + 6], x[8 * v + 7]));
}

template <typename TO>
__device__ __forceinline__ void load_row32_8(const TO *src, float (&x)[32]);
template <>
__device__ __forceinline__ void load_row32_8<float>(const float *src, float (&x)[32]) {
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
__device__ __forceinline__ void load_row32_8<__nv_bfloat16>(const __nv_bfloat16 *src, float (&x)[32]) {
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
    attn_f8_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                   const __nv_bfloat16 *__restrict__ q, AttnParams8 P) {
  extern __shared__ uint8_t smem_raw[];
  SmemLayout8 &sm =
      *reinterpret_cast<SmemLayout8 *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  volatile int *abort = &sm.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slot = blockIdx.x / P.q_tiles;
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
      mbar_init(&sm.s_free[s], 4);  // one arrival per softmax warp
      mbar_init(&sm.p_full[s], 4);
      mbar_init(&sm.pv_done[s], 1);
    }
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
    // ------------------------------------------------------------ producers: K8 (warp 0), V8 (warp 2)
    if (lane == 0) {
      const bool is_k = warp == 0;
      const int n_stages = is_k ? kStagesK : kStagesV;
      const CUtensorMap *map = is_k ? &tk : &tv;
      uint64_t *full = is_k ? sm.k_full : sm.v_full;
      uint64_t *empty = is_k ? sm.k_empty : sm.v_empty;
      uint32_t pend = 0, ph_bits = 0;
      TileIter8 it;
      it.start(sm.rng);
      for (int j = 0; j < P.n_tiles; ++j, it.next(sm.rng)) {
        const int st = j % n_stages;
        const uint32_t ph = (j / n_stages) & 1;
        if (!wait_parity(&empty[st], ph ^ 1, P.err, abort, is_k ? 41 : 42)) break;
        uint8_t *dst = is_k ? sm.k[st] : sm.v[st];
        mbar_arrive_expect_tx(&full[st], kTileBytes);
        if (is_k)
          tma_load_4d(dst, map, &full[st], 0, it.t0, h, b);            // 128 keys x 128 d bytes
        else
          tma_load_2d(dst, map, &full[st], it.t0, slot * kD);         // 128 d rows x 128 keys bytes
        pend |= 1u << st;
        ph_bits = (ph_bits & ~(1u << st)) | (ph << st);
      }
      if (*abort) {
        for (int st = 0; st < n_stages; ++st)
          if (pend & (1u << st)) wait_parity_drain(&full[st], (ph_bits >> st) & 1, P.err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = make_idesc(128, 128, 0, 0, 0);  // e4m3 A (TMEM) x e4m3 B (K-major), fp32 D
      uint64_t dk[kStagesK], dv[kStagesV];
#pragma unroll
      for (int st = 0; st < kStagesK; ++st) dk[st] = smem_desc_sw128(smem_u32(sm.k[st]), 16, 1024);
#pragma unroll
      for (int st = 0; st < kStagesV; ++st) dv[st] = smem_desc_sw128(smem_u32(sm.v[st]), 16, 1024);
      auto pick = [](const uint64_t *d, int n, int st) {
        uint64_t r = d[0];
#pragma unroll
        for (int i = 1; i < n; ++i) r = st == i ? d[i] : r;
        return r;
      };
      auto issue_s = [&](int j) {  // S_j = Q8 K8_j^T into S buffer j & 1: four K = 32 steps
        const uint64_t kd = pick(dk, kStagesK, j % kStagesK);
        const uint32_t d_s = tmem + kColS + (uint32_t)(j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < kD / 32; ++kk)
          mma_ts_f8(d_s, tmem + kColQ + (uint32_t)kk * 8, kd + (uint64_t)((kk * 32) >> 4), idesc, kk > 0 ? 1u : 0u);
        mma_commit(&sm.s_full[j & 1]);
        mma_commit(&sm.k_empty[j % kStagesK]);
      };
      auto issue_pv = [&](int j) {  // O (+)= P8_j V8_j: four K = 32-key steps
        const bool first = (j == 0) || (j == P.n_loc_tiles);
        const uint64_t vd = pick(dv, kStagesV, j % kStagesV);
        const uint32_t a_p = tmem + kColP + (uint32_t)(j & 1) * 32;
#pragma unroll
        for (int kk = 0; kk < kTileK / 32; ++kk)
          mma_ts_f8(tmem + kColO, a_p + kk * 8, vd + (uint64_t)((kk * 32) >> 4), idesc, (first && kk == 0) ? 0u : 1u);
        mma_commit(&sm.pv_done[j & 1]);
        mma_commit(&sm.v_empty[j % kStagesV]);
      };
      bool ok = wait_parity(&sm.q_ready, 0, P.err, abort, 50);
      for (int j = 0; ok && j < 2 && j < P.n_tiles; ++j) {
        ok = wait_parity(&sm.k_full[j % kStagesK], (j / kStagesK) & 1, P.err, abort, 51);
        if (!ok) break;
        tc_fence_after();
        issue_s(j);
      }
      for (int j = 0; ok && j < P.n_tiles; ++j) {
        const int jn = j + 2;
        if (jn < P.n_tiles) {  // S two tiles ahead, as soon as the softmax has read S_j
          ok = wait_parity(&sm.k_full[jn % kStagesK], (jn / kStagesK) & 1, P.err, abort, 52);
          if (ok) ok = wait_parity(&sm.s_free[j & 1], (uint32_t)(j >> 1) & 1, P.err, abort, 53);
          if (!ok) break;
          tc_fence_after();
          issue_s(jn);
        }
        ok = wait_parity(&sm.v_full[j % kStagesV], (j / kStagesV) & 1, P.err, abort, 54);
        if (ok) ok = wait_parity(&sm.p_full[j & 1], (uint32_t)(j >> 1) & 1, P.err, abort, 55);
        if (ok && j == P.n_loc_tiles) ok = wait_parity(&sm.o_free, 0, P.err, abort, 56);
        if (!ok) break;
        tc_fence_after();
        issue_pv(j);
      }
      if (!ok) {
        mma_commit(&sm.drain);
        wait_parity_drain(&sm.drain, 0, P.err);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int qrow = q0 + r;
    const bool row_ok = qrow < P.Lq;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const long long head_row = ((long long)b * P.Lq + (row_ok ? qrow : 0)) * P.H + h;
    TO *o_loc = reinterpret_cast<TO *>(P.o_loc) + head_row * kD;
    TO *o_hist = P.o_hist ? reinterpret_cast<TO *>(P.o_hist) + head_row * kD : nullptr;
    TO *o_full = P.o_full ? reinterpret_cast<TO *>(P.o_full) + head_row * kD : nullptr;
    const float amax_q = __uint_as_float(P.q_amax[slot]);
    const float inv_q = q8_inv(amax_q);
    const float c_log2 = P.scale_log2 * (amax_q / 448.f) * P.scale_k[slot];
    const float s_v = P.scale_v[slot];
    // Q8 row into TMEM: column c holds elements 4c .. 4c + 3 (lowest byte first)
    {
      const uint4 *src = reinterpret_cast<const uint4 *>(q + head_row * kD);
      uint32_t w8[32];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const uint4 v = row_ok ? __ldg(src + u) : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        float f[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 p = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
          f[2 * i] = p.x * inv_q;
          f[2 * i + 1] = p.y * inv_q;
        }
        w8[2 * u] = e4m3x4(f[0], f[1], f[2], f[3]);
        w8[2 * u + 1] = e4m3x4(f[4], f[5], f[6], f[7]);
      }
      tmem_st16(lane_base + kColQ, *reinterpret_cast<uint32_t(*)[16]>(&w8[0]));
      tmem_st16(lane_base + kColQ + 16, *reinterpret_cast<uint32_t(*)[16]>(&w8[16]));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.q_ready);
    }
    float m_ref = 0.f, l = 0.f, L_loc = -INFINITY;
    TileIter8 it;
    it.start(sm.rng);
    for (int j = 0; j < P.n_tiles; ++j, it.next(sm.rng)) {
      const bool grp_first = (j == 0) || (j == P.n_loc_tiles);
      const bool grp_last = (j == P.n_loc_tiles - 1) || (j == P.n_tiles - 1);
      const int lo = it.lo(sm.rng), hi = it.hi(sm.rng);
      const uint32_t col_s = kColS + (uint32_t)(j & 1) * 128;
      bool ok = wait_parity_spin(&sm.s_full[j & 1], (uint32_t)(j >> 1) & 1, P.err, abort, 61);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(lane_base + col_s + c * 32, sr[c]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.s_free[j & 1]);  // S_{j+2} may overwrite the buffer now
      if (lo > 0 || hi < kTileK) {     // keys of the tile outside the range
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c < lo || c >= hi) sr[c >> 5][c & 31] = 0xff800000u;
      }
      // p = 2^(t - m_ref + 6); l in fp32; P8 = e4m3(p), four per column (pairs on
      // the packed fp32 pipe: one FFMA2 and one FADD2 per two weights).  With
      // track_max the tile's maximum score is taken in the same pass.
      const float2 c2 = make_float2(c_log2, c_log2);
      uint32_t pk[32];
      auto weights = [&](float mref, bool track_max, float &mt) -> float {
        const float2 nm2 = make_float2(kPOffset - mref, kPOffset - mref);
        float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const uint32_t *row = &sr[c >> 3][(4 * c) & 31];
          const float s0 = __uint_as_float(row[0]), s1 = __uint_as_float(row[1]);
          const float s2 = __uint_as_float(row[2]), s3 = __uint_as_float(row[3]);
          if (track_max) {
            mx[c & 3] = fmax3f(mx[c & 3], s0, s1);
            mx[c & 3] = fmax3f(mx[c & 3], s2, s3);
          }
          const float2 x01 = ffma2f(make_float2(s0, s1), c2, nm2);
          const float2 x23 = ffma2f(make_float2(s2, s3), c2, nm2);
          const float2 p01 = make_float2(ex2f(x01.x), ex2f(x01.y));
          const float2 p23 = make_float2(ex2f(x23.x), ex2f(x23.y));
          ls[0] = fadd2f(ls[0], p01);
          ls[1] = fadd2f(ls[1], p23);
          pk[c] = e4m3x4(p01.x, p01.y, p23.x, p23.y);
        }
        if (track_max) mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * c_log2;
        return (ls[0].x + ls[0].y) + (ls[1].x + ls[1].y);
      };
      float l_tile, mt = 0.f;
      if (grp_first) {
        float mxs[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) mxs[t] = -INFINITY;
#pragma unroll
        for (int c = 0; c < 128; c += 2)
          mxs[(c >> 1) & 7] = fmax3f(mxs[(c >> 1) & 7], __uint_as_float(sr[c >> 5][c & 31]),
                                     __uint_as_float(sr[(c + 1) >> 5][(c + 1) & 31]));
        m_ref = fmax3f(fmax3f(mxs[0], mxs[1], mxs[2]), fmax3f(mxs[3], mxs[4], mxs[5]), fmaxf(mxs[6], mxs[7])) *
                c_log2;
        l = 0.f;
        l_tile = weights(m_ref, false, mt);
      } else {
        // weights against the current reference, the tile maximum alongside; the
        // reference moves (and the pass is redone) only when the maximum exceeds
        // it by more than kTau
        l_tile = weights(m_ref, true, mt);
        const bool moves = mt > m_ref + kTau;
        if (__any_sync(0xffffffffu, moves)) {
          // O (after PV_{j-1}) and l scale by 2^(m_ref - m_new)
          ok = wait_parity(&sm.pv_done[(j - 1) & 1], (uint32_t)((j - 1) >> 1) & 1, P.err, abort, 62);
          if (!__all_sync(0xffffffffu, ok)) break;
          tc_fence_after();
          const float m_new = moves ? mt : m_ref;
          const float f = ex2f(m_ref - m_new);
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
          l_tile = weights(m_ref, false, mt);
        }
      }
      l += l_tile;
      if (j >= 2) {  // PV_{j-2} has read this P buffer
        ok = wait_parity(&sm.pv_done[j & 1], (uint32_t)((j - 2) >> 1) & 1, P.err, abort, 63);
        if (!__all_sync(0xffffffffu, ok)) break;
      }
      tmem_st16(lane_base + kColP + (uint32_t)(j & 1) * 32, *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
      tmem_st16(lane_base + kColP + (uint32_t)(j & 1) * 32 + 16, *reinterpret_cast<uint32_t(*)[16]>(&pk[16]));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[j & 1]);

      if (!grp_last) continue;
      ok = wait_parity(&sm.pv_done[j & 1], (uint32_t)(j >> 1) & 1, P.err, abort, 64);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const bool is_loc = j < P.n_loc_tiles;
      const float inv_l = s_v / l;
      const float L = (m_ref - kPOffset + log2f(l)) * 0.69314718055994530942f;
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
        if (dst) store_row32_8<TO>(dst + c * 32, xo);
        if (write_full) {
          if (!is_loc) {
            float y[32];
            load_row32_8<TO>(o_loc + c * 32, y);
#pragma unroll
            for (int t = 0; t < 32; ++t) xo[t] = wa * y[t] + wb * xo[t];
          }
          store_row32_8<TO>(o_full + c * 32, xo);
        }
      }
      if (write_full && row_ok) P.l_full[head_row] = L_full;
      if (is_loc && !has_hist && row_ok) {
        if (o_hist) {
          const float zero[32] = {};
#pragma unroll 1
          for (int c = 0; c < 4; ++c) store_row32_8<TO>(o_hist + c * 32, zero);
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
ispa_status launch_typed8(const CUtensorMap &tk, const CUtensorMap &tv, const __nv_bfloat16 *q, const AttnParams8 &P,
                          int B, cudaStream_t s) {
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(attn_f8_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemBytes8);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(attn_f8_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kSmemBytes8);
    if (e != cudaSuccess) return cuda_status(e, "fp8 attention smem attribute");
    configured_device = dev;
  }
  attn_f8_kernel<TO><<<dim3(B * P.H * P.q_tiles), kThreads, kSmemBytes8, s>>>(tk, tv, q, P);
  note_launch();
  return cuda_status(cudaGetLastError(), "fp8 attention launch");
}

}  // namespace

size_t kv8_bytes(int B, int H, int Lkv) { return kv8_layout(B, H, Lkv).bytes; }

size_t attn_f8_workspace_bytes(int B, int H) { return a256((size_t)B * H * 4); }

ispa_status launch_kv8_prepare(int B, int H, int Lkv, int row_begin, int row_end, const void *k, const void *v,
                               void *kv8, cudaStream_t s) {
  const KV8Layout L = kv8_layout(B, H, Lkv);
  KV8State st = kv8_state(kv8, L, B, H);
  const bool reset = row_begin == 0;
  const size_t w = a256((size_t)B * H * 4);
  cudaError_t e = cudaSuccess;
  if (reset) e = cudaMemsetAsync(static_cast<char *>(kv8) + L.st_off, 0, 7 * w, s);
  if (e != cudaSuccess) return cuda_status(e, "fp8 K/V state clear");
  if (reset) {  // the transposed copy's pad columns stay zero
    e = cudaMemsetAsync(static_cast<char *>(kv8) + L.v_off, 0, (size_t)B * H * kD * L.Lkv_pad, s);
    if (e != cudaSuccess) return cuda_status(e, "fp8 V clear");
  }
  const int D = H * kD;
  const __nv_bfloat16 *kb = static_cast<const __nv_bfloat16 *>(k), *vb = static_cast<const __nv_bfloat16 *>(v);
  uint8_t *k8 = static_cast<uint8_t *>(kv8) + L.k_off, *v8t = static_cast<uint8_t *>(kv8) + L.v_off;
  const int rows = row_end - row_begin;
  const int BH = B * H;
  if (rows > 0) {
    const int vec = D / 8;
    const int want = std::max(1, (int)(((long long)rows * vec + 255) / 256));
    const int blocks = std::max((vec + 255) / 256, std::min(want, (sm_count() * 8 + B - 1) / B));
    amax_rows_kernel<<<dim3(blocks, B), 256, 0, s>>>(H, Lkv, row_begin, row_end, kb, st.cand_k);
    amax_rows_kernel<<<dim3(blocks, B), 256, 0, s>>>(H, Lkv, row_begin, row_end, vb, st.cand_v);
    note_launch(2);
  }
  kv8_decide_kernel<<<(BH + 255) / 256, 256, 0, s>>>(BH, reset ? 1 : 0, st);
  note_launch();
  auto convert = [&](int r0, int r1, int only_flagged) {
    if (r1 <= r0) return;
    const int vec = D / 16;
    const int want = std::max(1, (int)(((long long)(r1 - r0) * vec + 255) / 256));
    const int blocks = std::max((vec + 255) / 256, std::min(want, (sm_count() * 8 + B - 1) / B));
    k8_convert_kernel<<<dim3(blocks, B), 256, 0, s>>>(H, Lkv, r0, r1, only_flagged, kb, k8, st);
    v8t_convert_kernel<<<dim3((r1 - r0 + 63) / 64, H, B), 256, 0, s>>>(H, Lkv, L.Lkv_pad, r0, r1, only_flagged, vb,
                                                                       v8t, st);
    note_launch(2);
  };
  convert(row_begin, row_end, 0);
  if (!reset) convert(0, Lkv, 1);  // heads whose scale grew: every row again
  return cuda_status(cudaGetLastError(), "fp8 K/V prepare launch");
}

ispa_status launch_attn_f8(const ispa_attn_desc &d, const GroupRanges &g, float scale, const void *q,
                           const void *kv8, void *o_loc, float *l_loc, void *o_hist, float *l_hist, void *o_full,
                           float *l_full, void *workspace, cudaStream_t s) {
  if (g.Lq == 0) return ISPA_OK;
  AttnParams8 P{};
  ispa_status st = device_err(&P.err);
  if (st != ISPA_OK) return st;
  const int D = d.H * kD;
  const KV8Layout L = kv8_layout(d.B, d.H, g.Lkv);
  const KV8State kst = kv8_state(const_cast<void *>(kv8), L, d.B, d.H);
  unsigned int *q_amax = static_cast<unsigned int *>(workspace);
  cudaError_t e = cudaMemsetAsync(q_amax, 0, (size_t)d.B * d.H * 4, s);
  if (e != cudaSuccess) return cuda_status(e, "fp8 attention workspace clear");
  {
    const int vec = D / 8;
    const int want = std::max(1, (int)(((long long)g.Lq * vec + 255) / 256));
    const int blocks = std::max((vec + 255) / 256, std::min(want, (sm_count() * 8 + d.B - 1) / d.B));
    amax_rows_kernel<<<dim3(blocks, d.B), 256, 0, s>>>(d.H, g.Lq, 0, g.Lq, static_cast<const __nv_bfloat16 *>(q),
                                                       q_amax);
    note_launch();
  }
  CUtensorMap tk, tv;
  {
    const uint64_t dims[4] = {(uint64_t)kD, (uint64_t)g.Lkv, (uint64_t)d.H, (uint64_t)d.B};
    const uint64_t strides[3] = {(uint64_t)D, (uint64_t)kD, (uint64_t)D * (uint64_t)g.Lkv};
    const uint32_t box[4] = {kD, 128, 1, 1};
    if ((st = make_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, static_cast<const char *>(kv8) + L.k_off, dims,
                        strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != ISPA_OK)
      return st;
  }
  {
    const uint64_t dims[2] = {(uint64_t)L.Lkv_pad, (uint64_t)d.B * d.H * kD};
    const uint64_t strides[1] = {(uint64_t)L.Lkv_pad};
    const uint32_t box[2] = {128, 128};
    if ((st = make_tmap(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, static_cast<const char *>(kv8) + L.v_off, dims,
                        strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != ISPA_OK)
      return st;
  }
  P.H = d.H;
  P.Lq = g.Lq;
  P.q_tiles = (g.Lq + kTileQ - 1) / kTileQ;
  auto tiles = [](int lo, int hi) { return (hi - (lo - lo % kAlign) + kTileK - 1) / kTileK; };
  for (int r = 0; r < g.n_loc; ++r) {
    P.r_begin[P.n_ranges] = g.loc_begin[r];
    P.r_end[P.n_ranges] = g.loc_end[r];
    P.n_loc_tiles += tiles(g.loc_begin[r], g.loc_end[r]);
    ++P.n_ranges;
  }
  P.n_loc_ranges = P.n_ranges;
  P.n_tiles = P.n_loc_tiles;
  if (g.hist_end > g.hist_begin) {
    P.r_begin[P.n_ranges] = g.hist_begin;
    P.r_end[P.n_ranges] = g.hist_end;
    P.n_tiles += tiles(g.hist_begin, g.hist_end);
    ++P.n_ranges;
  }
  P.scale_log2 = scale * 1.4426950408889634f;
  P.q_amax = q_amax;
  P.scale_k = kst.scale_k;
  P.scale_v = kst.scale_v;
  P.o_loc = o_loc;
  P.o_hist = o_hist;
  P.o_full = o_full;
  P.l_loc = l_loc;
  P.l_hist = l_hist;
  P.l_full = l_full;
  const __nv_bfloat16 *qb = static_cast<const __nv_bfloat16 *>(q);
  if (d.out_dtype == ISPA_F32) return launch_typed8<float>(tk, tv, qb, P, d.B, s);
  return launch_typed8<__nv_bfloat16>(tk, tv, qb, P, d.B, s);
}

}  // namespace ispa
