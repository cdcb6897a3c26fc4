// gemm_tc.cuh -- tcgen05 GEMM building block (sm_100a).
//
// D[128 x 256 tile] = sum over K of A_tile * B_tile, accumulated in tensor
// memory (128 lanes x 256 fp32 columns), with operands staged by TMA into
// 128-byte-swizzled shared memory through a 4-stage mbarrier pipeline.  The
// 256-wide tile halves the A traffic per FLOP against a 128-wide one (1.75x the
// rate measured on a large bf16 product).
//
// Warp roles (192 threads):
//   warp 0      TMA producer (one elected lane)
//   warp 1      TMEM allocator + MMA issuer (one elected lane)
//   warps 2..5  epilogue: tcgen05.ld of the accumulator rows, then the
//               problem-specific store (each thread owns one output row)
//
// Operand staging.  An A tile is 16 KB and a B tile 32 KB: 128 (A) or 256 (B)
// rows of M or N by one 128-byte swizzle span of K for K-major operands, or BK
// rows of K by 128 / 256 M or N elements (128-byte column blocks) for MN-major
// operands.  Per stage the MMA warp issues 4 instructions of K = 8 (tf32),
// K = 16 (bf16) or K = 32 (e4m3 / int8, K-major only).  The copy engine's time
// is mostly per box, so a stage arrives in as few boxes as the layout allows:
// the K-major B tile as one 256-row box, an MN-major operand through a 3D
// view whose third dimension is its column blocks (map_mn_blocked).
//
// Store epilogues go through shared memory (the operand stages are idle once
// the accumulator is complete) so that each row is written by a whole warp.
//
// Up to two sub-problems that share A (same M, K) but have different B and
// outputs run in one launch: blockIdx.x enumerates the tiles of problem 0,
// then those of problem 1.  Tiles may be restricted to the upper triangle
// (used for the symmetric Gram matrix).
//
// fp32-accurate products on the tf32 pipe (split3): with x = x_hi + x_lo,
// x_hi the nearest tf32 and x_lo the remainder, A B is taken as
// A_hi B_hi + A_hi B_lo + A_lo B_hi, three passes over the K range into one
// accumulator (the dropped A_lo B_lo is below fp32 rounding).  For these
// products the K range of a tile may be cut to a triangle of A (lower:
// k < m0 + BM; upper: k >= m0) and split into chunks of chunk_kt K-tiles, one
// CTA each (blockIdx.x = tile * nchunk + chunk; an empty chunk exits at once),
// whose partial products are added to the output with atomics.  The tensor
// cores accumulate in fp32 with truncation, a bias of about 2^-25 of the sum
// per MMA step: fine for the solve, not for quantities that are small
// differences of large sums.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace ispa {
namespace tcg {

constexpr int BM = 128, BN = 256, STAGES = 4;
constexpr int TILE_BYTES = BM * 128;    // A tile: 128 rows x 128 bytes of K
constexpr int TILE_B_BYTES = BN * 128;  // B tile: 256 rows x 128 bytes of K
constexpr int SMEM_BYTES = STAGES * (TILE_BYTES + TILE_B_BYTES) + 1024 /*align*/ + 256 /*barriers*/;
constexpr int THREADS = 192;

enum Epi : int {
  EPI_STORE_F32 = 0,      // out = acc
  EPI_STORE_TF32_SQ = 1,  // out = tf32_rn(acc); r2 += sum acc^2
  EPI_ACCUM_F32 = 2,      // out += acc
  EPI_STORE_BF16 = 3,     // out = bf16_rn(acc)
  EPI_ATOMIC_F32 = 4,     // out += acc with atomics (split K)
  EPI_SCALED = 5          // out = acc * row_scale[m] * col_scale[n], bf16 or fp32 (out_bf16)
};

enum Tri : int { TRI_NONE = 0, TRI_A_LOWER = 1, TRI_A_UPPER = 2 };

struct SubProblem {
  int N;          // columns of this problem's output
  int tiles_n;    // ceil(N / BN)
  int upper;      // 1: only tiles/elements with row <= col
  int epi;        // Epi
  void *out;      // [M, N] row-major, ld = ldo
  long long ldo;
  int b_blk;      // 1: B's map delivers a whole stage in one box (see the operand staging note)
};

struct Params {
  int M, K;
  int tiles_m;
  int n_tiles0;   // tiles of problem 0 (upper-triangle filter already applied)
  int n_tiles;    // tiles of both problems (the grid size)
  int kind_tf32;  // 1: kind::tf32 (fp32 operands), 0: kind::f16 with bf16 operands
  int kind_f8;    // 8-bit K-major operands: 1 = e4m3 (kind::f8f6f4), 2 = int8 (kind::i8, int32 accumulator)
  int a_mn, b_mn; // operand majorness (1 = MN-major)
  int a_blk;      // 1: A's map delivers a whole stage in one box
  uint32_t idesc;
  double *r2;     // EPI_STORE_TF32_SQ accumulator
  const float *row_scale, *col_scale;  // EPI_SCALED factors
  int out_bf16;   // EPI_SCALED: bf16 output (else fp32)
  int split3;     // 1: three passes (hi hi, hi lo, lo hi) with the lo maps
  int tri;        // Tri: K range of a tile cut to a triangle of A
  int nchunk;     // K chunks per tile (0 or 1: none)
  int chunk_kt;   // K-tiles per chunk
  SubProblem p[2];
  DevErr err;
};

// Enumerates upper-triangle tiles (tile row tm <= tile col tn covering some i <= j).
__host__ __device__ inline int upper_tile_count(int tiles_m, int tiles_n) {
  int c = 0;
  for (int tm = 0; tm < tiles_m; ++tm) {
    const int first = (tm * BM) / BN;  // first tile column whose block has a col >= row
    c += tiles_n > first ? tiles_n - first : 0;
  }
  return c;
}

__device__ inline void tile_coords(const Params &P, int t, int &prob, int &tm, int &tn) {
  prob = t < P.n_tiles0 ? 0 : 1;
  if (prob == 1) t -= P.n_tiles0;
  const SubProblem &sp = P.p[prob];
  if (!sp.upper) {
    tm = t / sp.tiles_n;
    tn = t - tm * sp.tiles_n;
    return;
  }
  for (tm = 0; tm < P.tiles_m; ++tm) {
    const int first = (tm * BM) / BN;
    const int cnt = sp.tiles_n > first ? sp.tiles_n - first : 0;
    if (t < cnt) {
      tn = first + t;
      return;
    }
    t -= cnt;
  }
  tn = 0;
}

__device__ __forceinline__ void red_add_v4(float *p, float4 v) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
}

template <int EPI>
__device__ __forceinline__ void epilogue_chunk(const Params &P, const SubProblem &sp, int row, int col0,
                                               const uint32_t (&r)[32], double &sq) {
  if (row >= P.M) return;
  const int N = sp.N;
  if (EPI == EPI_SCALED) {
    const float rs = P.row_scale[row];
    float x[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float acc = P.kind_f8 == 2 ? __int2float_rn((int)r[j]) : __uint_as_float(r[j]);
      x[j] = col0 + j < N ? acc * rs * P.col_scale[col0 + j] : 0.f;
    }
    if (P.out_bf16) {
      __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(sp.out) + (long long)row * sp.ldo + col0;
      if (col0 + 32 <= N && (reinterpret_cast<uintptr_t>(o) & 15) == 0) {
        uint4 *o4 = reinterpret_cast<uint4 *>(o);
#pragma unroll
        for (int v = 0; v < 4; ++v)
          o4[v] = make_uint4(pack_bf16x2(x[8 * v], x[8 * v + 1]), pack_bf16x2(x[8 * v + 2], x[8 * v + 3]),
                             pack_bf16x2(x[8 * v + 4], x[8 * v + 5]), pack_bf16x2(x[8 * v + 6], x[8 * v + 7]));
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (col0 + j < N) o[j] = __float2bfloat16_rn(x[j]);
      }
    } else {
      float *o = reinterpret_cast<float *>(sp.out) + (long long)row * sp.ldo + col0;
      if (col0 + 32 <= N && (reinterpret_cast<uintptr_t>(o) & 15) == 0) {
#pragma unroll
        for (int v = 0; v < 8; ++v)
          reinterpret_cast<float4 *>(o)[v] = make_float4(x[4 * v], x[4 * v + 1], x[4 * v + 2], x[4 * v + 3]);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (col0 + j < N) o[j] = x[j];
      }
    }
    return;
  }
  if (EPI == EPI_STORE_BF16) {
    __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(sp.out) + (long long)row * sp.ldo + col0;
    if (col0 + 32 <= N) {
      uint4 *o4 = reinterpret_cast<uint4 *>(o);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        uint4 w;
        w.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
        w.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
        w.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
        w.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
        o4[v] = w;
      }
    } else {
      for (int j = 0; j < 32 && col0 + j < N; ++j) o[j] = __float2bfloat16_rn(__uint_as_float(r[j]));
    }
    return;
  }
  float *o = reinterpret_cast<float *>(sp.out) + (long long)row * sp.ldo + col0;
  const bool full = col0 + 32 <= N && (!sp.upper || col0 >= row) && (reinterpret_cast<uintptr_t>(o) & 15) == 0;
  if (full) {
    float4 *o4 = reinterpret_cast<float4 *>(o);
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      float4 x = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]), __uint_as_float(r[4 * v + 2]),
                             __uint_as_float(r[4 * v + 3]));
      if (EPI == EPI_ATOMIC_F32) {
        red_add_v4(o + 4 * v, x);
        continue;
      }
      if (EPI == EPI_STORE_TF32_SQ) {
        sq += (double)x.x * x.x + (double)x.y * x.y + (double)x.z * x.z + (double)x.w * x.w;
        x = make_float4(to_tf32_rn(x.x), to_tf32_rn(x.y), to_tf32_rn(x.z), to_tf32_rn(x.w));
      }
      if (EPI == EPI_ACCUM_F32) {
        const float4 y = o4[v];
        x.x += y.x;
        x.y += y.y;
        x.z += y.z;
        x.w += y.w;
      }
      o4[v] = x;
    }
  } else {
    for (int j = 0; j < 32; ++j) {
      const int c = col0 + j;
      if (c >= N) break;
      if (sp.upper && c < row) continue;
      float x = __uint_as_float(r[j]);
      if (EPI == EPI_ATOMIC_F32) {
        atomicAdd(o + j, x);
        continue;
      }
      if (EPI == EPI_STORE_TF32_SQ) {
        sq += (double)x * x;
        x = to_tf32_rn(x);
      }
      if (EPI == EPI_ACCUM_F32) x += o[j];
      o[j] = x;
    }
  }
}

// Store epilogue through shared memory, for the plain stores (bf16 or fp32),
// the scaled 8-bit one, the accumulating one (out += acc, only i <= j for an
// upper-triangle problem) and the tf32-rounding one with its sum of squares,
// with N % 16 == 0 and 16-byte aligned rows.  Each
// epilogue warp owns 32 rows of the tile: it moves its accumulator rows out
// of tensor memory (lane = row), writes them to its own staging area in
// 16-byte chunks (chunk j of row r at slot j ^ r, so that neither the row-wise
// writes nor the column-wise reads below collide in a bank), then writes the
// rows back one at a time with the whole warp: 512 (bf16) or 1024 (fp32)
// contiguous bytes per row, instead of every store instruction touching 32
// rows.  The staging areas reuse the operand stages, idle once the
// accumulator is complete.
enum StageMode { STAGE_STORE = 0, STAGE_SCALED = 1, STAGE_ACCUM = 2, STAGE_TF32_SQ = 3 };

template <bool BF16_OUT, int MODE>
__device__ __forceinline__ void epilogue_staged(const Params &P, const SubProblem &sp, uint32_t tmem_rows, int quarter,
                                                int lane, int m0, int n0, uint8_t *stage, double &sq) {
  constexpr bool SCALED = MODE == STAGE_SCALED;
  constexpr int ELEM = BF16_OUT ? 2 : 4;
  constexpr int CPR = BN * ELEM / 16;  // 16-byte chunks per row
  const int N = sp.N;
  const int row = m0 + quarter * 32 + lane;
  const float rs = SCALED && row < P.M ? P.row_scale[row] : 1.f;
  const int n_chunks = min(BN, N - n0 + 31) / 32;
  uint8_t *my = stage + lane * (CPR * 16);
  for (int c = 0; c < BN / 32; ++c) {
    uint32_t r[32];
    tmem_ld32(tmem_rows + c * 32, r);
    tmem_wait_ld();
    if (c >= n_chunks) continue;
    float cs = 1.f;
    if (SCALED) {
      const int col = n0 + c * 32 + lane;
      cs = col < N ? P.col_scale[col] : 0.f;
    }
    float x[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float acc = SCALED && P.kind_f8 == 2 ? __int2float_rn((int)r[j]) : __uint_as_float(r[j]);
      x[j] = SCALED ? acc * rs * __shfl_sync(0xffffffffu, cs, j) : acc;
      if (MODE == STAGE_TF32_SQ) {
        if (row < P.M && n0 + c * 32 + j < N) sq += (double)acc * acc;
        x[j] = to_tf32_rn(acc);
      }
    }
    if (BF16_OUT) {
#pragma unroll
      for (int v = 0; v < 4; ++v)
        *reinterpret_cast<uint4 *>(my + (((c * 4 + v) ^ lane) * 16)) =
            make_uint4(pack_bf16x2(x[8 * v], x[8 * v + 1]), pack_bf16x2(x[8 * v + 2], x[8 * v + 3]),
                       pack_bf16x2(x[8 * v + 4], x[8 * v + 5]), pack_bf16x2(x[8 * v + 6], x[8 * v + 7]));
    } else {
#pragma unroll
      for (int v = 0; v < 8; ++v)
        *reinterpret_cast<float4 *>(my + (((c * 8 + v) ^ lane) * 16)) =
            make_float4(x[4 * v], x[4 * v + 1], x[4 * v + 2], x[4 * v + 3]);
    }
  }
  __syncwarp();
  for (int rr = 0; rr < 32; ++rr) {
    const int grow = m0 + quarter * 32 + rr;
    if (grow >= P.M) break;
    const uint8_t *src = stage + rr * (CPR * 16);
    uint8_t *dst = static_cast<uint8_t *>(sp.out) + ((long long)grow * sp.ldo + n0) * ELEM;
#pragma unroll
    for (int j = lane; j < CPR; j += 32) {
      const int col = n0 + j * (16 / ELEM);
      if (col >= N) continue;
      uint4 v = *reinterpret_cast<const uint4 *>(src + ((j ^ rr) * 16));
      if (MODE == STAGE_ACCUM) {  // fp32: old + acc, acc taken as 0 left of the diagonal of an upper problem
        const float4 old = *reinterpret_cast<const float4 *>(dst + j * 16);
        const float a[4] = {__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z), __uint_as_float(v.w)};
        const float o4[4] = {old.x, old.y, old.z, old.w};
        float s4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) s4[e] = (sp.upper && col + e < grow) ? o4[e] : o4[e] + a[e];
        v = make_uint4(__float_as_uint(s4[0]), __float_as_uint(s4[1]), __float_as_uint(s4[2]), __float_as_uint(s4[3]));
      }
      *reinterpret_cast<uint4 *>(dst + j * 16) = v;
    }
  }
}

#ifdef ISPA_DEFINE_GEMM_KERNEL
// tma maps: ta = A operand; tb[prob] = B operand of each sub-problem; with
// split3, ta_lo and tb_lo hold the remainders of A and of B (problem 0 only).
__global__ void __launch_bounds__(THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb0,
                const __grid_constant__ CUtensorMap tb1, const __grid_constant__ CUtensorMap ta_lo,
                const __grid_constant__ CUtensorMap tb_lo, Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + STAGES * TILE_BYTES;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * (TILE_BYTES + TILE_B_BYTES));
  uint64_t *empty = full + STAGES;
  uint64_t *done = empty + STAGES;
  uint64_t *drain = done + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nchunk = P.nchunk > 1 ? P.nchunk : 1;
  int prob, tm, tn;
  tile_coords(P, blockIdx.x / nchunk, prob, tm, tn);
  const SubProblem &sp = P.p[prob];
  const CUtensorMap *tB = prob == 0 ? &tb0 : &tb1;
  const int m0 = tm * BM, n0 = tn * BN;
  const int bk = P.kind_tf32 ? 32 : (P.kind_f8 ? 128 : 64);  // K elements per stage (128 bytes)
  // this CTA's K-tiles [kt_begin, kt_end): the tile's range (cut to A's
  // triangle), then this chunk of it
  int kt_begin = 0, kt_end = (P.K + bk - 1) / bk;
  if (P.tri == TRI_A_LOWER) kt_end = min(kt_end, (m0 + BM + bk - 1) / bk);
  if (P.tri == TRI_A_UPPER) kt_begin = m0 / bk;
  if (nchunk > 1) {
    kt_begin += (blockIdx.x % nchunk) * P.chunk_kt;
    kt_end = min(kt_end, kt_begin + P.chunk_kt);
  }
  if (kt_begin >= kt_end) return;  // empty chunk: nothing to add (before any barrier or TMEM)
  const int k_span = kt_end - kt_begin;
  const int k_tiles = k_span * (P.split3 ? 3 : 1);  // pipeline iterations
  const int e128 = bk;                          // elements per 128-byte row
  const uint32_t kstep_kmajor = 32;             // bytes per MMA K-step inside a K-major row
  const uint32_t kstep_mn = P.kind_tf32 ? 1024 : 2048;  // bytes per MMA K-step in an MN-major tile
  const uint32_t mn_box_bytes = (uint32_t)bk * 128;     // one 128-byte-wide MN-major box

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    mbar_init(done, 1);
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&ta);
    tma_prefetch_desc(tB);
    if (P.split3) {
      tma_prefetch_desc(&ta_lo);
      tma_prefetch_desc(&tb_lo);
    }
  }
  if (warp == 1) tmem_alloc(tmem_slot, BN);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t pending = 0;  // bit s: a load into stage s may still be in flight
      uint32_t issued_phase = 0;
      for (int kt = 0; kt < k_tiles; ++kt) {
        const int s = kt % STAGES;
        const uint32_t ph = (kt / STAGES) & 1;
        if (!wait_parity(empty + s, ph ^ 1, P.err, abort, 1)) break;
        mbar_arrive_expect_tx(full + s, TILE_BYTES + TILE_B_BYTES);
        const int pass = kt / k_span;  // split3: 0 = hi hi, 1 = hi lo, 2 = lo hi
        const int k0 = (kt_begin + kt - pass * k_span) * bk;
        const CUtensorMap *mA = pass == 2 ? &ta_lo : &ta;
        const CUtensorMap *mB = pass == 1 ? &tb_lo : tB;
        uint8_t *a = sA + s * TILE_BYTES;
        uint8_t *b = sB + s * TILE_B_BYTES;
        if (!P.a_mn) {
          tma_load_2d(a, mA, full + s, k0, m0);
        } else if (P.a_blk) {  // 3D map: (element in block, k, block of e128)
          tma_load_3d(a, mA, full + s, 0, k0, m0 / e128);
        } else {
          for (int c = 0; c < BM / e128; ++c) tma_load_2d(a + c * mn_box_bytes, mA, full + s, m0 + c * e128, k0);
        }
        if (!P.b_mn) {
          if (sp.b_blk) {  // one 256-row box
            tma_load_2d(b, mB, full + s, k0, n0);
          } else {         // 128-row boxes, one after the other
            for (int c = 0; c < BN / 128; ++c) tma_load_2d(b + c * TILE_BYTES, mB, full + s, k0, n0 + c * 128);
          }
        } else if (sp.b_blk) {
          tma_load_3d(b, mB, full + s, 0, k0, n0 / e128);
        } else {
          for (int c = 0; c < BN / e128; ++c) tma_load_2d(b + c * mn_box_bytes, mB, full + s, n0 + c * e128, k0);
        }
        pending |= 1u << s;
        issued_phase = (issued_phase & ~(1u << s)) | (ph << s);
      }
      if (*abort) {
        for (int s = 0; s < STAGES; ++s)
          if (pending & (1u << s)) wait_parity_drain(full + s, (issued_phase >> s) & 1, P.err);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = true;
      for (int kt = 0; kt < k_tiles; ++kt) {
        const int s = kt % STAGES;
        const uint32_t ph = (kt / STAGES) & 1;
        if (!wait_parity(full + s, ph, P.err, abort, 2)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_base = smem_u32(sA + s * TILE_BYTES);
        const uint32_t b_base = smem_u32(sB + s * TILE_B_BYTES);
        // MN-major: bf16 uses 8-row SWIZZLE_128B atoms (SBO = 1024 B between them),
        // tf32 uses 4-row SWIZZLE_128B_BASE32B atoms (SBO = 512 B).
        const uint32_t mn_layout = P.kind_tf32 ? 1u : 2u;
        const uint32_t mn_sbo = P.kind_tf32 ? 512u : 1024u;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t ad = P.a_mn ? smem_desc(a_base + ks * kstep_mn, mn_box_bytes, mn_sbo, mn_layout)
                                     : smem_desc_sw128(a_base + ks * kstep_kmajor, 16, 1024);
          const uint64_t bd = P.b_mn ? smem_desc(b_base + ks * kstep_mn, mn_box_bytes, mn_sbo, mn_layout)
                                     : smem_desc_sw128(b_base + ks * kstep_kmajor, 16, 1024);
          mma_ss(tmem, ad, bd, P.idesc, (kt > 0 || ks > 0) ? 1u : 0u, P.kind_f8 ? P.kind_f8 + 1 : P.kind_tf32);
        }
        mma_commit(empty + s);
      }
      mma_commit(ok ? done : drain);
      if (!ok) wait_parity_drain(drain, 0, P.err);
    }
  } else {
    // epilogue warps 2..5: TMEM lane quarter = warp % 4
    const int quarter = warp & 3;
    const int row = m0 + quarter * 32 + lane;
    double sq = 0.0;
    const bool staged = (sp.epi == EPI_STORE_BF16 || sp.epi == EPI_STORE_F32 || sp.epi == EPI_SCALED ||
                         sp.epi == EPI_ACCUM_F32 || sp.epi == EPI_STORE_TF32_SQ) &&
                        sp.N % 16 == 0 && sp.ldo % 16 == 0 && (reinterpret_cast<uintptr_t>(sp.out) & 15) == 0;
    const uint32_t tmem_rows = tmem + ((uint32_t)(quarter * 32) << 16);
    uint8_t *stage = smem + quarter * (32 * BN * 4);  // 32 KB per warp inside the operand stages
    if (staged) {
      if (wait_parity(done, 0, P.err, abort, 3)) {
        tc_fence_after();
        const bool bf16_out = sp.epi == EPI_STORE_BF16 || (sp.epi == EPI_SCALED && P.out_bf16);
        if (sp.epi == EPI_SCALED) {
          if (bf16_out) epilogue_staged<true, STAGE_SCALED>(P, sp, tmem_rows, quarter, lane, m0, n0, stage, sq);
          else epilogue_staged<false, STAGE_SCALED>(P, sp, tmem_rows, quarter, lane, m0, n0, stage, sq);
        } else if (sp.epi == EPI_ACCUM_F32) {
          epilogue_staged<false, STAGE_ACCUM>(P, sp, tmem_rows, quarter, lane, m0, n0, stage, sq);
        } else if (sp.epi == EPI_STORE_TF32_SQ) {
          epilogue_staged<false, STAGE_TF32_SQ>(P, sp, tmem_rows, quarter, lane, m0, n0, stage, sq);
        } else {
          if (bf16_out) epilogue_staged<true, STAGE_STORE>(P, sp, tmem_rows, quarter, lane, m0, n0, stage, sq);
          else epilogue_staged<false, STAGE_STORE>(P, sp, tmem_rows, quarter, lane, m0, n0, stage, sq);
        }
      }
    } else if (wait_parity(done, 0, P.err, abort, 3)) {
      tc_fence_after();
      const int n_chunks = min(BN, sp.N - n0 + 31) / 32;
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + c * 32, r);
        tmem_wait_ld();
        if (c >= n_chunks) continue;
        switch (sp.epi) {
          case EPI_STORE_F32: epilogue_chunk<EPI_STORE_F32>(P, sp, row, n0 + c * 32, r, sq); break;
          case EPI_STORE_TF32_SQ: epilogue_chunk<EPI_STORE_TF32_SQ>(P, sp, row, n0 + c * 32, r, sq); break;
          case EPI_ACCUM_F32: epilogue_chunk<EPI_ACCUM_F32>(P, sp, row, n0 + c * 32, r, sq); break;
          case EPI_ATOMIC_F32: epilogue_chunk<EPI_ATOMIC_F32>(P, sp, row, n0 + c * 32, r, sq); break;
          case EPI_SCALED: epilogue_chunk<EPI_SCALED>(P, sp, row, n0 + c * 32, r, sq); break;
          default: epilogue_chunk<EPI_STORE_BF16>(P, sp, row, n0 + c * 32, r, sq); break;
        }
      }
    }
    if (sp.epi == EPI_STORE_TF32_SQ) {
      sq = warp_sum_d(sq);
      if (lane == 0 && P.r2) atomicAdd(P.r2, sq);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, BN);
}
#endif  // ISPA_DEFINE_GEMM_KERNEL

}  // namespace tcg

// fp32 map of a row-major [outer, inner] matrix with leading dimension ld
// (elements, a multiple of 4).  K-major operands use the 128-byte swizzle;
// MN-major tf32 operands the 128-byte swizzle with 32-byte atoms.
inline ispa_status map2d_f32_ld(CUtensorMap *m, const void *base, int inner, int outer, long long ld, int box_inner,
                                int box_outer, bool mn_major) {
  const uint64_t dims[2] = {(uint64_t)inner, (uint64_t)outer};
  const uint64_t strides[1] = {(uint64_t)ld * 4};
  const uint32_t box[2] = {(uint32_t)box_inner, (uint32_t)box_outer};
  return make_tmap(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box,
                   mn_major ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B);
}

// Blocked view of an MN-major operand, so that one TMA load fills a whole
// stage.  The copy engine spends a roughly fixed time per box (a 4 KB box
// moves at a third of the rate of a 32 KB one), and an MN-major stage of
// 128-byte-wide column blocks would otherwise take one box per block.  The
// row-major [outer, inner] matrix (leading dimension ld elements of elem
// bytes, inner = M or N) is seen as three dimensions: the e128 elements of a
// 128-byte block, the outer (K) rows, and the blocks, whose stride (128 bytes)
// is smaller than the row stride; the box {e128, box_k, blocks} lands in
// shared memory as blocks one after the other, the layout of the per-block
// boxes.  Only when inner is a whole number of blocks and holds at least one
// box of them (else *blocked = false and the caller keeps per-block boxes).
inline ispa_status map_mn_blocked(CUtensorMap *m, CUtensorMapDataType dt, int elem, const void *base, int inner,
                                  int outer, long long ld, int box_k, int blocks, CUtensorMapSwizzle sw,
                                  bool *blocked) {
  const int e128 = 128 / elem;
  *blocked = inner % e128 == 0 && inner / e128 >= blocks;
  if (!*blocked) return ISPA_OK;
  const uint64_t dims[3] = {(uint64_t)e128, (uint64_t)outer, (uint64_t)(inner / e128)};
  const uint64_t strides[2] = {(uint64_t)ld * elem, 128};
  const uint32_t box[3] = {(uint32_t)e128, (uint32_t)box_k, (uint32_t)blocks};
  return make_tmap(m, dt, 3, base, dims, strides, box, sw);
}

// MN-major fp32 operand map for a tile of `blocks` 32-element blocks: blocked
// when possible, per-block 2D boxes otherwise.
inline ispa_status map_f32_mn(CUtensorMap *m, const void *base, int inner, int outer, long long ld, int box_k,
                              int blocks, int *blk) {
  bool b = false;
  ispa_status st = map_mn_blocked(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, inner, outer, ld, box_k, blocks,
                                  CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B, &b);
  if (st != ISPA_OK) return st;
  *blk = b ? 1 : 0;
  return b ? ISPA_OK : map2d_f32_ld(m, base, inner, outer, ld, 32, box_k, true);
}

inline ispa_status map2d_f32(CUtensorMap *m, const void *base, int inner, int outer, int box_inner, int box_outer,
                             bool mn_major) {
  return map2d_f32_ld(m, base, inner, outer, inner, box_inner, box_outer, mn_major);
}

// Host launchers (gemm_tc.cu).  launch_tc_gemm: up to two sub-problems, one
// pass.  launch_tc_gemm_split3: one sub-problem, fp32-accurate three-pass
// product from the hi and lo maps of A and B.
ispa_status launch_tc_gemm(const CUtensorMap &ta, const CUtensorMap &tb0, const CUtensorMap &tb1,
                           tcg::Params &P, cudaStream_t s);
ispa_status launch_tc_gemm_split3(const CUtensorMap &ta, const CUtensorMap &ta_lo, const CUtensorMap &tb,
                                  const CUtensorMap &tb_lo, tcg::Params &P, cudaStream_t s);
}  // namespace ispa
