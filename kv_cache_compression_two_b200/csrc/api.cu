// api.cu -- the extern "C" entry points of libispa: argument validation,
// group-range normalisation, error reporting and dispatch to the kernels.
#include <math.h>
#include <mutex>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "internal.h"

// Per-device error word: [0] ispa_status of the first device-side failure, [1] its detail.
__device__ int g_ispa_device_error[2];

#include <atomic>

namespace ispa {

static thread_local char t_last_error[512] = "";
static std::atomic<unsigned long long> g_launches{0};

void note_launch(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

ispa_status fail(ispa_status st, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_error, sizeof(t_last_error), fmt, ap);
  va_end(ap);
  return st;
}

ispa_status cuda_status(cudaError_t e, const char *what) {
  if (e == cudaSuccess) return ISPA_OK;
  return fail(ISPA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
int *g_err_addr[kMaxDevices] = {};
int g_sms[kMaxDevices] = {};
long long g_wait_limit_ns = 2000000000LL;  // 2 s per device-side wait

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

CtxGetCurrentFn ctx_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}
}  // namespace

void *current_context() {
  CtxGetCurrentFn fn = ctx_fn();
  CUcontext c = nullptr;
  if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

namespace {
void *g_err_ctx[kMaxDevices] = {};
}  // namespace

ispa_status device_err(DevErr *out) {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return fail(ISPA_ERR_CUDA, "no current CUDA device");
  std::lock_guard<std::mutex> lock(g_mu);
  // looked up again whenever the thread's current context is not the one the
  // cached address belongs to (a reset device has a new context and module)
  void *ctx = current_context();
  if (!g_err_addr[dev] || !ctx || ctx != g_err_ctx[dev]) {
    void *p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_ispa_device_error);
    if (e != cudaSuccess) return cuda_status(e, "cudaGetSymbolAddress(error word)");
    g_err_addr[dev] = static_cast<int *>(p);
    g_err_ctx[dev] = current_context();
  }
  out->word = g_err_addr[dev];
  out->limit_ns = g_wait_limit_ns;
  return ISPA_OK;
}

int sm_count() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 148;
  if (!g_sms[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    g_sms[dev] = n > 0 ? n : 148;
  }
  return g_sms[dev];
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

ispa_status make_tmap(CUtensorMap *m, CUtensorMapDataType dt, int rank, const void *base, const uint64_t *dims,
                      const uint64_t *strides_bytes, const uint32_t *box, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(ISPA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint64_t d[5], st[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) st[i] = strides_bytes[i];
  CUresult r = fn(m, dt, (cuuint32_t)rank, const_cast<void *>(base), d, st, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ISPA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return ISPA_OK;
}

}  // namespace ispa

using namespace ispa;

namespace {

bool dtype_ok(ispa_dtype d) { return d == ISPA_F32 || d == ISPA_BF16; }

// Validates an attention descriptor and turns frame ranges into token ranges.
ispa_status attn_ranges(const ispa_attn_desc *d, GroupRanges *g, float *scale) {
  if (!d) return fail(ISPA_ERR_INVALID_ARG, "desc is NULL");
  if (d->B < 1 || d->H < 1 || d->tokens_per_frame < 1)
    return fail(ISPA_ERR_INVALID_ARG, "B, H and tokens_per_frame must be >= 1");
  if (d->head_dim != 32 && d->head_dim != 64 && d->head_dim != 128)
    return fail(ISPA_ERR_INVALID_ARG, "head_dim must be 32, 64 or 128 (got %d)", d->head_dim);
  if (!dtype_ok(d->in_dtype) || !dtype_ok(d->out_dtype)) return fail(ISPA_ERR_INVALID_ARG, "bad dtype");
  if (d->v_layout != ISPA_V_PLAIN && d->v_layout != ISPA_V_F16_PREPARED && d->v_layout != ISPA_KV_E4M3_PREPARED)
    return fail(ISPA_ERR_INVALID_ARG, "bad v_layout");
  if (d->v_layout != ISPA_V_PLAIN && (d->in_dtype != ISPA_BF16 || d->head_dim != 128))
    return fail(ISPA_ERR_INVALID_ARG, "a prepared V (fp16) or K/V (fp8) goes with bf16 inputs and head_dim 128");
  const int F = d->kv_frames;
  if (F < 1) return fail(ISPA_ERR_INVALID_ARG, "kv_frames must be >= 1");
  if (d->sink_frames < 0 || d->sink_frames > F) return fail(ISPA_ERR_INVALID_ARG, "sink_frames out of [0, kv_frames]");
  if (!(0 <= d->cur_begin && d->cur_begin < d->cur_end && d->cur_end <= F))
    return fail(ISPA_ERR_INVALID_ARG, "current chunk [%d, %d) invalid for kv_frames %d", d->cur_begin, d->cur_end, F);
  if (!(0 <= d->hist_begin && d->hist_begin <= d->hist_end && d->hist_end <= F))
    return fail(ISPA_ERR_INVALID_ARG, "history [%d, %d) invalid for kv_frames %d", d->hist_begin, d->hist_end, F);
  const bool hist = d->hist_end > d->hist_begin;
  if (hist && (d->hist_begin < d->sink_frames || (d->hist_begin < d->cur_end && d->cur_begin < d->hist_end)))
    return fail(ISPA_ERR_INVALID_ARG, "history group overlaps the local group");
  const long long tpf = d->tokens_per_frame;
  if ((long long)F * tpf > (1LL << 30) || (long long)d->B * F * tpf * d->H * d->head_dim > (1LL << 40))
    return fail(ISPA_ERR_INVALID_ARG, "tensor too large");
  // local = [0, S) u [cb, ce), merged when they touch
  int lb[2], le[2], n = 0;
  const int S = d->sink_frames, cb = d->cur_begin, ce = d->cur_end;
  if (S > 0) {
    if (cb <= S) {
      lb[n] = 0;
      le[n++] = ce > S ? ce : S;
    } else {
      lb[n] = 0;
      le[n++] = S;
      lb[n] = cb;
      le[n++] = ce;
    }
  } else {
    lb[n] = cb;
    le[n++] = ce;
  }
  g->n_loc = n;
  for (int i = 0; i < n; ++i) {
    g->loc_begin[i] = (int)(lb[i] * tpf);
    g->loc_end[i] = (int)(le[i] * tpf);
  }
  g->hist_begin = (int)(d->hist_begin * tpf);
  g->hist_end = (int)(d->hist_end * tpf);
  g->q_begin = (int)(cb * tpf);
  g->Lq = (int)((ce - cb) * tpf);
  g->Lkv = (int)(F * tpf);
  *scale = d->softmax_scale > 0.f ? d->softmax_scale : 1.f / sqrtf((float)d->head_dim);
  if (!isfinite(*scale)) return fail(ISPA_ERR_INVALID_ARG, "softmax_scale must be finite");
  return ISPA_OK;
}

bool ptr_ok(const void *p) { return p != nullptr && aligned16(p); }

// Eviction (gather: full layout of desc -> compact layout of the evicted desc)
// and restore (scatter back).  Validates desc, alignment and overlap.
ispa_status kv_remap(const ispa_attn_desc *desc, const void *k, const void *v, void *k_out, void *v_out, bool gather,
                     cudaStream_t s) {
  GroupRanges g;
  float scale;
  ispa_status st = attn_ranges(desc, &g, &scale);
  if (st != ISPA_OK) return st;
  if (desc->v_layout == ISPA_KV_E4M3_PREPARED)
    return fail(ISPA_ERR_INVALID_ARG, "a prepared fp8 K/V is not evicted or restored: move the bf16 K/V and "
                "prepare the result (ispa_kv8_prepare)");
  if (!ptr_ok(k) || !ptr_ok(v) || !ptr_ok(k_out) || !ptr_ok(v_out))
    return fail(ISPA_ERR_INVALID_ARG, "the four K/V pointers must be 16-byte aligned device pointers");
  const long long esize = desc->in_dtype == ISPA_BF16 ? 2 : 4;
  const long long row_bytes = (long long)desc->H * desc->head_dim * esize;  // a multiple of 64
  const long long full_rows = g.Lkv;
  const long long len0 = g.loc_end[0] - g.loc_begin[0];
  const long long kept_rows = len0 + (g.n_loc > 1 ? g.loc_end[1] - g.loc_begin[1] : 0);
  const long long full_bytes = desc->B * full_rows * row_bytes, kept_bytes = desc->B * kept_rows * row_bytes;
  const long long in_bytes = gather ? full_bytes : kept_bytes, out_bytes = gather ? kept_bytes : full_bytes;
  // a prepared V is longer than K by its per-head state, which moves with it
  const bool prepared = desc->v_layout == ISPA_V_F16_PREPARED;
  const long long v_in_bytes =
      prepared ? (long long)v16_bytes(desc->B, desc->H, (int)(gather ? full_rows : kept_rows)) : in_bytes;
  const long long v_out_bytes =
      prepared ? (long long)v16_bytes(desc->B, desc->H, (int)(gather ? kept_rows : full_rows)) : out_bytes;
  auto overlap = [](const void *a, long long na, const void *b, long long nb) {
    const char *x = (const char *)a, *y = (const char *)b;
    return x < y + nb && y < x + na;
  };
  if (overlap(k_out, out_bytes, k, in_bytes) || overlap(k_out, out_bytes, v, v_in_bytes) ||
      overlap(v_out, v_out_bytes, k, in_bytes) || overlap(v_out, v_out_bytes, v, v_in_bytes) ||
      overlap(k_out, out_bytes, v_out, v_out_bytes))
    return fail(ISPA_ERR_INVALID_ARG, "the outputs must not overlap each other or the inputs");
  st = launch_kv_remap(desc->B, full_rows, kept_rows, g.loc_begin[0], len0, g.n_loc > 1 ? g.loc_begin[1] : 0,
                       row_bytes, gather, k, v, k_out, v_out, s);
  if (st != ISPA_OK || desc->v_layout != ISPA_V_F16_PREPARED) return st;
  // a prepared V carries its per-head state (exponent, 2^-e, range statistics) along
  const int in_rows = (int)(gather ? full_rows : kept_rows), out_rows = (int)(gather ? kept_rows : full_rows);
  const char *src = static_cast<const char *>(v) + v16_state_offset(desc->B, desc->H, in_rows);
  char *dst = static_cast<char *>(v_out) + v16_state_offset(desc->B, desc->H, out_rows);
  return cuda_status(cudaMemcpyAsync(dst, src, v16_state_bytes(desc->B, desc->H), cudaMemcpyDeviceToDevice, s),
                     "prepared V state copy");
}

}  // namespace

extern "C" {

const char *ispa_version(void) { return "ispa-b200 0.1 (sm_100a)"; }

const char *ispa_last_error(void) { return t_last_error; }

uint64_t ispa_launch_count(void) { return (uint64_t)g_launches.load(std::memory_order_relaxed); }

ispa_status ispa_check_device_error(ispa_stream_t stream, int *detail) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_status(e, "stream synchronize");
  DevErr de;
  ispa_status st = device_err(&de);
  if (st != ISPA_OK) return st;
  int host[2] = {0, 0};
  e = cudaMemcpy(host, de.word, sizeof(host), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_status(e, "read device error word");
  if (host[0] != 0) {
    const int zero[2] = {0, 0};
    cudaMemcpy(de.word, zero, sizeof(zero), cudaMemcpyHostToDevice);
  }
  if (detail) *detail = host[1];
  if (host[0] == ISPA_ERR_NOT_SPD) return fail(ISPA_ERR_NOT_SPD, "G + lambda I is not positive definite (pivot %d)", host[1]);
  if (host[0] == ISPA_ERR_TIMEOUT) return fail(ISPA_ERR_TIMEOUT, "device-side wait timed out (site %d)", host[1]);
  if (host[0] != 0) return fail(ISPA_ERR_CUDA, "device error code %d", host[0]);
  return ISPA_OK;
}

size_t ispa_attn_split_workspace_bytes(const ispa_attn_desc *desc) {
  GroupRanges g;
  float scale;
  if (attn_ranges(desc, &g, &scale) != ISPA_OK) return 0;
  if (desc->in_dtype != ISPA_BF16) return 0;
  return attn_tc_workspace_bytes(desc->B, desc->H, g.Lkv, desc->v_layout);
}

ispa_status ispa_attn_split(const ispa_attn_desc *desc, const void *q, const void *k, const void *v, void *o_loc,
                            float *lse_loc, void *o_hist, float *lse_hist, void *o_full, float *lse_full,
                            void *workspace, size_t workspace_bytes, ispa_stream_t stream) {
  GroupRanges g;
  float scale;
  ispa_status st = attn_ranges(desc, &g, &scale);
  if (st != ISPA_OK) return st;
  const size_t need = ispa_attn_split_workspace_bytes(desc);
  if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace)))
    return fail(ISPA_ERR_INVALID_ARG, "workspace needs %zu bytes (16-byte aligned)", need);
  if (!ptr_ok(q) || !ptr_ok(k) || (!ptr_ok(v) && desc->v_layout != ISPA_KV_E4M3_PREPARED))
    return fail(ISPA_ERR_INVALID_ARG, "q, k, v must be 16-byte aligned device pointers");
  if (!ptr_ok(o_loc) || !ptr_ok(lse_loc)) return fail(ISPA_ERR_INVALID_ARG, "o_loc and lse_loc are required (16-byte aligned)");
  if ((o_hist == nullptr) != (lse_hist == nullptr)) return fail(ISPA_ERR_INVALID_ARG, "o_hist and lse_hist: both or neither");
  if ((o_full == nullptr) != (lse_full == nullptr)) return fail(ISPA_ERR_INVALID_ARG, "o_full and lse_full: both or neither");
  if ((o_hist && !ptr_ok(o_hist)) || (lse_hist && !ptr_ok(lse_hist)) || (o_full && !ptr_ok(o_full)) ||
      (lse_full && !ptr_ok(lse_full)))
    return fail(ISPA_ERR_INVALID_ARG, "outputs must be 16-byte aligned");
  if (desc->in_dtype == ISPA_BF16) {
    if (desc->head_dim != 128) return fail(ISPA_ERR_UNSUPPORTED, "bf16 attention is compiled for head_dim 128 only");
    return launch_attn_tc(*desc, g, scale, q, k, v, o_loc, lse_loc, o_hist, lse_hist, o_full, lse_full, workspace,
                          (cudaStream_t)stream);
  }
  return launch_attn_simt(*desc, g, scale, (const float *)q, (const float *)k, (const float *)v, o_loc, lse_loc, o_hist,
                          lse_hist, o_full, lse_full, (cudaStream_t)stream);
}

size_t ispa_v16_bytes(const ispa_attn_desc *desc) {
  GroupRanges g;
  float scale;
  if (attn_ranges(desc, &g, &scale) != ISPA_OK) return 0;
  if (desc->in_dtype != ISPA_BF16 || desc->head_dim != 128) return 0;
  return v16_bytes(desc->B, desc->H, g.Lkv);
}

ispa_status ispa_v16_prepare(const ispa_attn_desc *desc, const void *v, int frame_begin, int frame_end, void *v16,
                             ispa_stream_t stream) {
  GroupRanges g;
  float scale;
  ispa_status st = attn_ranges(desc, &g, &scale);
  if (st != ISPA_OK) return st;
  if (desc->in_dtype != ISPA_BF16 || desc->head_dim != 128)
    return fail(ISPA_ERR_UNSUPPORTED, "a prepared fp16 V is built for bf16 inputs with head_dim 128");
  if (!(0 <= frame_begin && frame_begin <= frame_end && frame_end <= desc->kv_frames))
    return fail(ISPA_ERR_INVALID_ARG, "frames [%d, %d) invalid for kv_frames %d", frame_begin, frame_end,
                desc->kv_frames);
  if (!ptr_ok(v) || !ptr_ok(v16)) return fail(ISPA_ERR_INVALID_ARG, "v and v16 must be 16-byte aligned device pointers");
  const long long tpf = desc->tokens_per_frame;
  const char *a = static_cast<const char *>(v), *b = static_cast<const char *>(v16);
  const long long vb = (long long)desc->B * g.Lkv * desc->H * 128 * 2, v16b = (long long)v16_bytes(desc->B, desc->H, g.Lkv);
  if (a < b + v16b && b < a + vb) return fail(ISPA_ERR_INVALID_ARG, "v16 must not overlap v");
  return launch_v16_prepare(desc->B, desc->H, g.Lkv, (int)(frame_begin * tpf), (int)(frame_end * tpf), v, v16,
                            (cudaStream_t)stream);
}

size_t ispa_kv8_bytes(const ispa_attn_desc *desc) {
  GroupRanges g;
  float scale;
  if (attn_ranges(desc, &g, &scale) != ISPA_OK) return 0;
  if (desc->in_dtype != ISPA_BF16 || desc->head_dim != 128) return 0;
  return kv8_bytes(desc->B, desc->H, g.Lkv);
}

ispa_status ispa_kv8_prepare(const ispa_attn_desc *desc, const void *k, const void *v, int frame_begin,
                             int frame_end, void *kv8, ispa_stream_t stream) {
  GroupRanges g;
  float scale;
  ispa_status st = attn_ranges(desc, &g, &scale);
  if (st != ISPA_OK) return st;
  if (desc->in_dtype != ISPA_BF16 || desc->head_dim != 128)
    return fail(ISPA_ERR_UNSUPPORTED, "a prepared fp8 K/V is built for bf16 inputs with head_dim 128");
  if (!(0 <= frame_begin && frame_begin <= frame_end && frame_end <= desc->kv_frames))
    return fail(ISPA_ERR_INVALID_ARG, "frames [%d, %d) invalid for kv_frames %d", frame_begin, frame_end,
                desc->kv_frames);
  if (!ptr_ok(k) || !ptr_ok(v) || !ptr_ok(kv8))
    return fail(ISPA_ERR_INVALID_ARG, "k, v and kv8 must be 16-byte aligned device pointers");
  const long long nb = (long long)desc->B * g.Lkv * desc->H * 128 * 2, n8 = (long long)kv8_bytes(desc->B, desc->H, g.Lkv);
  auto overlap = [](const void *a, long long na, const void *b, long long nbb) {
    const char *x = (const char *)a, *y = (const char *)b;
    return x < y + nbb && y < x + na;
  };
  if (overlap(kv8, n8, k, nb) || overlap(kv8, n8, v, nb)) return fail(ISPA_ERR_INVALID_ARG, "kv8 must not overlap k or v");
  const long long tpf = desc->tokens_per_frame;
  return launch_kv8_prepare(desc->B, desc->H, g.Lkv, (int)(frame_begin * tpf), (int)(frame_end * tpf), k, v, kv8,
                            (cudaStream_t)stream);
}

ispa_status ispa_lse_merge(int rows, int H, int head_dim, ispa_dtype o_dtype, const void *o_a, const float *lse_a,
                           const void *o_b, const float *lse_b, void *o_out, float *lse_out, ispa_stream_t stream) {
  if (rows < 0 || H < 1 || head_dim < 8 || head_dim % 8 != 0 || !dtype_ok(o_dtype))
    return fail(ISPA_ERR_INVALID_ARG, "rows >= 0, H >= 1, head_dim a positive multiple of 8");
  if (rows == 0) return ISPA_OK;
  if (o_dtype == ISPA_F32 && head_dim % 4 != 0) return fail(ISPA_ERR_INVALID_ARG, "head_dim");
  if (!ptr_ok(o_a) || !ptr_ok(o_b) || !ptr_ok(o_out) || !lse_a || !lse_b || !lse_out)
    return fail(ISPA_ERR_INVALID_ARG, "pointers must be non-NULL, O pointers 16-byte aligned");
  const size_t n = (size_t)rows * H;
  const char *lo = (const char *)lse_out;
  auto overlap = [&](const float *p) { return lo < (const char *)(p + n) && (const char *)p < lo + n * 4; };
  if (overlap(lse_a) || overlap(lse_b)) return fail(ISPA_ERR_INVALID_ARG, "lse_out must not overlap lse_a or lse_b");
  return launch_lse_merge(rows, H, head_dim, o_dtype, o_a, lse_a, o_b, lse_b, o_out, lse_out, (cudaStream_t)stream);
}

size_t ispa_accum_stats_workspace_bytes(int T, int D, int Dout, ispa_precision prec) {
  if (T < 0 || D < 1 || Dout < 1) return 0;
  return stats_workspace_bytes(T, D, Dout, prec);
}

ispa_status ispa_accum_stats(int T, int D, int Dout, const float *a_loc, const float *a_full, const float *W, float *G,
                             float *C, double *r2, ispa_precision prec, void *workspace, size_t workspace_bytes,
                             ispa_stream_t stream) {
  if (T < 0 || D < 1 || Dout < 1) return fail(ISPA_ERR_INVALID_ARG, "T >= 0, D >= 1, Dout >= 1");
  if (prec != ISPA_PREC_TF32 && prec != ISPA_PREC_F32) return fail(ISPA_ERR_INVALID_ARG, "bad precision");
  if (prec == ISPA_PREC_TF32 && (D % 32 != 0 || Dout % 32 != 0))
    return fail(ISPA_ERR_INVALID_ARG, "ISPA_PREC_TF32 needs D and Dout multiples of 32");
  if ((long long)T * D > (1LL << 34) || (long long)D * Dout > (1LL << 31))
    return fail(ISPA_ERR_INVALID_ARG, "sizes too large");
  if (!ptr_ok(a_loc) || !ptr_ok(a_full) || !ptr_ok(W) || !ptr_ok(G) || !ptr_ok(C) || !r2)
    return fail(ISPA_ERR_INVALID_ARG, "pointers must be non-NULL and 16-byte aligned");
  if (T == 0) return ISPA_OK;
  const size_t need = stats_workspace_bytes(T, D, Dout, prec);
  if (!workspace || workspace_bytes < need || !aligned16(workspace))
    return fail(ISPA_ERR_INVALID_ARG, "workspace needs %zu bytes (16-byte aligned)", need);
  return launch_stats(T, D, Dout, a_loc, a_full, W, G, C, r2, prec, workspace, (cudaStream_t)stream);
}

namespace {
size_t round256(size_t x) { return (x + 255) & ~size_t(255); }
}  // namespace

size_t ispa_warmup_fused_workspace_bytes(const ispa_attn_desc *desc, int Dout) {
  GroupRanges g;
  float scale;
  if (!desc || Dout < 1 || attn_ranges(desc, &g, &scale) != ISPA_OK) return 0;
  const int T = desc->B * g.Lq, D = desc->H * desc->head_dim;
  return round256(stats_workspace_bytes(T, D, Dout, ISPA_PREC_TF32)) + round256((size_t)T * desc->H * 4) +
         attn_tc_workspace_bytes(desc->B, desc->H, g.Lkv, desc->v_layout);
}

ispa_status ispa_warmup_fused(const ispa_attn_desc *desc, const void *q, const void *k, const void *v,
                              const float *W, int Dout, float *o_full, float *l_full, float *G, float *C,
                              double *r2, void *workspace, size_t workspace_bytes, ispa_stream_t stream) {
  GroupRanges g;
  float scale;
  ispa_status st = attn_ranges(desc, &g, &scale);
  if (st != ISPA_OK) return st;
  if (desc->in_dtype != ISPA_BF16 || desc->head_dim != 128)
    return fail(ISPA_ERR_UNSUPPORTED, "the fused warmup is compiled for bf16 inputs with head_dim 128");
  if (desc->v_layout == ISPA_KV_E4M3_PREPARED)
    return fail(ISPA_ERR_UNSUPPORTED, "the fused warmup runs the bf16 attention (fp8 K/V is a post-switch layout)");
  const int D = desc->H * desc->head_dim;
  const long long T = (long long)desc->B * g.Lq;
  if (Dout < 32 || Dout % 32 != 0) return fail(ISPA_ERR_INVALID_ARG, "Dout must be a positive multiple of 32");
  if (T * D > (1LL << 34) || (long long)D * Dout > (1LL << 31)) return fail(ISPA_ERR_INVALID_ARG, "sizes too large");
  if (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(v) || !ptr_ok(W) || !ptr_ok(o_full) || !ptr_ok(l_full) || !ptr_ok(G) ||
      !ptr_ok(C) || !r2)
    return fail(ISPA_ERR_INVALID_ARG, "pointers must be non-NULL and 16-byte aligned");
  const size_t need = ispa_warmup_fused_workspace_bytes(desc, Dout);
  if (!workspace || workspace_bytes < need || !aligned16(workspace))
    return fail(ISPA_ERR_INVALID_ARG, "workspace needs %zu bytes (16-byte aligned)", need);
  if (T == 0) return ISPA_OK;
  ispa_attn_desc d = *desc;
  d.out_dtype = ISPA_F32;
  char *w = static_cast<char *>(workspace);
  const size_t stats_bytes = round256(stats_workspace_bytes((int)T, D, Dout, ISPA_PREC_TF32));
  float *lse_loc = reinterpret_cast<float *>(w + stats_bytes);
  void *attn_ws = w + stats_bytes + round256((size_t)T * d.H * 4);
  float *dA = nullptr, *Ar = nullptr;
  stats_row_operands(w, (int)T, D, Dout, &dA, &Ar);
  cudaStream_t s = (cudaStream_t)stream;
  // O_loc goes to the statistics' Ar buffer (left there rounded to tf32), dA next to it
  st = launch_attn_tc(d, g, scale, q, k, v, Ar, lse_loc, nullptr, nullptr, o_full, l_full, attn_ws, s, dA);
  if (st != ISPA_OK) return st;
  return launch_stats((int)T, D, Dout, nullptr, nullptr, W, G, C, r2, ISPA_PREC_TF32, w, s, true);
}

size_t ispa_ridge_workspace_bytes(int D, int Dout) {
  if (D < 1 || Dout < 1) return 0;
  return ridge_workspace_bytes(D, Dout);
}

ispa_status ispa_ridge_solve(int D, int Dout, const float *G, const float *C, const double *r2, float lambda,
                             int lambda_relative, int refine_steps, float *dW, double *eps, void *workspace,
                             size_t workspace_bytes, ispa_stream_t stream) {
  if (D < 1 || Dout < 1 || D > 32768 || (long long)D * Dout > (1LL << 31))
    return fail(ISPA_ERR_INVALID_ARG, "1 <= D <= 32768, Dout >= 1");
  if (!(lambda >= 0.f) || !isfinite(lambda)) return fail(ISPA_ERR_INVALID_ARG, "lambda must be finite and >= 0");
  if (refine_steps < 0 || refine_steps > 16) return fail(ISPA_ERR_INVALID_ARG, "refine_steps in [0, 16]");
  if (!ptr_ok(G) || !ptr_ok(C) || !r2 || !ptr_ok(dW) || !eps)
    return fail(ISPA_ERR_INVALID_ARG, "pointers must be non-NULL, matrices 16-byte aligned");
  const size_t need = ridge_workspace_bytes(D, Dout);
  if (!workspace || workspace_bytes < need || !aligned16(workspace))
    return fail(ISPA_ERR_INVALID_ARG, "workspace needs %zu bytes (16-byte aligned)", need);
  return launch_ridge(D, Dout, G, C, r2, lambda, lambda_relative, refine_steps, dW, eps, workspace,
                      (cudaStream_t)stream);
}

ispa_status ispa_ridge_solve_noalloc(int D, int Dout, const float *G, const float *C, const double *r2, float lambda,
                                     int lambda_relative, int refine_steps, float *dW, double *eps,
                                     ispa_stream_t stream) {
  if (D < 1 || Dout < 1 || D > ISPA_RIDGE_NOALLOC_MAX_D || Dout > ISPA_RIDGE_NOALLOC_MAX_DOUT)
    return fail(ISPA_ERR_INVALID_ARG,
                "ispa_ridge_solve_noalloc: need 1 <= D <= %d and 1 <= Dout <= %d (got D=%d, Dout=%d); use "
                "ispa_ridge_solve with a workspace for larger sizes",
                ISPA_RIDGE_NOALLOC_MAX_D, ISPA_RIDGE_NOALLOC_MAX_DOUT, D, Dout);
  if (!(lambda >= 0.f) || !isfinite(lambda)) return fail(ISPA_ERR_INVALID_ARG, "lambda must be finite and >= 0");
  if (refine_steps < 0 || refine_steps > 16) return fail(ISPA_ERR_INVALID_ARG, "refine_steps in [0, 16]");
  if (!ptr_ok(G) || !ptr_ok(C) || !r2 || !ptr_ok(dW) || !eps)
    return fail(ISPA_ERR_INVALID_ARG, "pointers must be non-NULL, matrices 16-byte aligned");
  void *scratch = nullptr;
  ispa_status st = ridge_noalloc_scratch(D, Dout, &scratch);
  if (st != ISPA_OK) return st;
  return launch_ridge(D, Dout, G, C, r2, lambda, lambda_relative, refine_steps, dW, eps, scratch,
                      (cudaStream_t)stream);
}

size_t ispa_absorb_error_workspace_bytes(int D, int Dout) {
  if (D < 1 || Dout < 1) return 0;
  return absorb_error_workspace_bytes(D, Dout);
}

ispa_status ispa_absorb_error(int D, int Dout, const float *G, const float *C, const double *r2, const float *dW,
                              double *eps, void *workspace, size_t workspace_bytes, ispa_stream_t stream) {
  if (D < 1 || Dout < 1 || (long long)D * Dout > (1LL << 31)) return fail(ISPA_ERR_INVALID_ARG, "bad D, Dout");
  if (!ptr_ok(G) || !ptr_ok(C) || !r2 || !ptr_ok(dW) || !eps)
    return fail(ISPA_ERR_INVALID_ARG, "pointers must be non-NULL, matrices 16-byte aligned");
  const size_t need = absorb_error_workspace_bytes(D, Dout);
  if (!workspace || workspace_bytes < need || !aligned16(workspace))
    return fail(ISPA_ERR_INVALID_ARG, "workspace needs %zu bytes (16-byte aligned)", need);
  return launch_absorb_error(D, Dout, G, C, r2, dW, eps, workspace, (cudaStream_t)stream);
}

ispa_status ispa_select_layers(int N, const double *eps, int K, unsigned char *is_local, int *idx,
                               ispa_stream_t stream) {
  if (N < 0 || N > 4096 || K < 0 || K > N) return fail(ISPA_ERR_INVALID_ARG, "need 0 <= K <= N <= 4096");
  if (N == 0) return ISPA_OK;
  if (!eps || !is_local || (K > 0 && !idx)) return fail(ISPA_ERR_INVALID_ARG, "NULL pointer");
  return launch_select(N, eps, K, is_local, idx, (cudaStream_t)stream);
}

ispa_status ispa_absorb_weight(int D, int Dout, const void *W, ispa_dtype w_dtype, const float *dW, void *W_new,
                               ispa_dtype out_dtype, ispa_stream_t stream) {
  if (D < 1 || Dout < 1 || ((long long)D * Dout) % 4 != 0 || (long long)D * Dout > (1LL << 34))
    return fail(ISPA_ERR_INVALID_ARG, "D * Dout must be a positive multiple of 4");
  if (!dtype_ok(w_dtype) || !dtype_ok(out_dtype)) return fail(ISPA_ERR_INVALID_ARG, "bad dtype");
  if (!ptr_ok(W) || !ptr_ok(dW) || !ptr_ok(W_new)) return fail(ISPA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (W_new == W && w_dtype != out_dtype) return fail(ISPA_ERR_INVALID_ARG, "in-place needs matching dtypes");
  return launch_absorb_weight(D, Dout, W, w_dtype, dW, W_new, out_dtype, (cudaStream_t)stream);
}

size_t ispa_attn_local_proj_workspace_bytes(const ispa_attn_desc *desc) {
  GroupRanges g;
  float scale;
  if (attn_ranges(desc, &g, &scale) != ISPA_OK) return 0;
  const size_t a = (size_t)desc->B * g.Lq * desc->H * desc->head_dim * 2;
  const size_t l = (size_t)desc->B * g.Lq * desc->H * 4;
  return ((a + 255) & ~size_t(255)) + ((l + 255) & ~size_t(255)) +
         attn_tc_workspace_bytes(desc->B, desc->H, g.Lkv, desc->v_layout);
}

ispa_status ispa_attn_local_proj(const ispa_attn_desc *desc, const void *q, const void *k, const void *v,
                                 const void *W_proj, int Dout, void *y, ispa_dtype y_dtype, void *workspace,
                                 size_t workspace_bytes, ispa_stream_t stream) {
  GroupRanges g;
  float scale;
  ispa_status st = attn_ranges(desc, &g, &scale);
  if (st != ISPA_OK) return st;
  if (desc->in_dtype != ISPA_BF16 || desc->head_dim != 128)
    return fail(ISPA_ERR_UNSUPPORTED, "post-switch projection is compiled for bf16 inputs with head_dim 128");
  if (Dout < 16 || Dout % 16 != 0) return fail(ISPA_ERR_INVALID_ARG, "Dout must be a positive multiple of 16");
  if (!dtype_ok(y_dtype)) return fail(ISPA_ERR_INVALID_ARG, "bad y dtype");
  if (!ptr_ok(q) || !ptr_ok(k) || (!ptr_ok(v) && desc->v_layout != ISPA_KV_E4M3_PREPARED) || !ptr_ok(W_proj) ||
      !ptr_ok(y))
    return fail(ISPA_ERR_INVALID_ARG, "pointers must be non-NULL and 16-byte aligned");
  const size_t need = ispa_attn_local_proj_workspace_bytes(desc);
  if (!workspace || workspace_bytes < need || !aligned16(workspace))
    return fail(ISPA_ERR_INVALID_ARG, "workspace needs %zu bytes (16-byte aligned)", need);
  ispa_attn_desc d = *desc;
  d.hist_begin = d.hist_end = 0;
  d.out_dtype = ISPA_BF16;
  g.hist_begin = g.hist_end = 0;
  const size_t a_bytes = (((size_t)d.B * g.Lq * d.H * d.head_dim * 2) + 255) & ~size_t(255);
  const size_t l_bytes = (((size_t)d.B * g.Lq * d.H * 4) + 255) & ~size_t(255);
  void *a_loc = workspace;
  float *lse = reinterpret_cast<float *>(static_cast<char *>(workspace) + a_bytes);
  void *attn_ws = static_cast<char *>(workspace) + a_bytes + l_bytes;
  st = launch_attn_tc(d, g, scale, q, k, v, a_loc, lse, nullptr, nullptr, nullptr, nullptr, attn_ws,
                      (cudaStream_t)stream);
  if (st != ISPA_OK) return st;
  const int D = d.H * d.head_dim;
  return launch_gemm_bf16(d.B * g.Lq, Dout, D, a_loc, W_proj, y, y_dtype, (cudaStream_t)stream);
}

namespace {

bool q8_ok(ispa_q8_format f) { return f == ISPA_Q8_E4M3 || f == ISPA_Q8_INT8; }

bool q8_k_ok(int K) { return K >= 16 && K % 16 == 0; }

// int8 products accumulate exactly in int32: |sum| <= K * 127^2 must stay below 2^31
constexpr int kQ8Int8MaxK = 131072;

// [a, a + na) and [b, b + nb) (bytes) overlap
bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
  const char *x = static_cast<const char *>(a), *y = static_cast<const char *>(b);
  return x < y + nb && y < x + na;
}

}  // namespace

ispa_status ispa_quantize_rows(int M, int K, const void *x, ispa_q8_format fmt, void *q, float *sa,
                               ispa_stream_t stream) {
  if (M < 0 || !q8_k_ok(K)) return fail(ISPA_ERR_INVALID_ARG, "need M >= 0 and K a positive multiple of 16");
  if (!q8_ok(fmt)) return fail(ISPA_ERR_INVALID_ARG, "bad 8-bit format");
  if (M == 0) return ISPA_OK;
  if (!ptr_ok(x) || !ptr_ok(q) || !ptr_ok(sa)) return fail(ISPA_ERR_INVALID_ARG, "pointers must be non-NULL and 16-byte aligned");
  const size_t xb = (size_t)M * K * 2, qb = (size_t)M * K, sb = (size_t)M * 4;
  if (overlaps(x, xb, q, qb) || overlaps(x, xb, sa, sb) || overlaps(q, qb, sa, sb))
    return fail(ISPA_ERR_INVALID_ARG, "x, q and sa must not overlap");
  return launch_quant_rows(M, K, x, fmt, q, sa, (cudaStream_t)stream);
}

ispa_status ispa_quantize_weight(int K, int N, const void *W, ispa_q8_format fmt, void *qT, float *sw,
                                 ispa_stream_t stream) {
  if (N < 0 || !q8_k_ok(K)) return fail(ISPA_ERR_INVALID_ARG, "need N >= 0 and K a positive multiple of 16");
  if (!q8_ok(fmt)) return fail(ISPA_ERR_INVALID_ARG, "bad 8-bit format");
  if (N == 0) return ISPA_OK;
  if (!ptr_ok(W) || !ptr_ok(qT) || !ptr_ok(sw)) return fail(ISPA_ERR_INVALID_ARG, "pointers must be non-NULL and 16-byte aligned");
  const size_t wb = (size_t)K * N * 2, qb = (size_t)K * N, sb = (size_t)N * 4;
  if (overlaps(W, wb, qT, qb) || overlaps(W, wb, sw, sb) || overlaps(qT, qb, sw, sb))
    return fail(ISPA_ERR_INVALID_ARG, "W, qT and sw must not overlap");
  return launch_quant_cols(K, N, W, fmt, qT, sw, (cudaStream_t)stream);
}

ispa_status ispa_gemm_bf16(int M, int N, int K, const void *A, const void *W, void *y, ispa_dtype y_dtype,
                           ispa_stream_t stream) {
  if (M < 0 || N < 0 || N % 16 != 0 || K < 16 || K % 16 != 0)
    return fail(ISPA_ERR_INVALID_ARG, "need M >= 0, N a multiple of 16 and K a positive multiple of 16");
  if (!dtype_ok(y_dtype)) return fail(ISPA_ERR_INVALID_ARG, "bad y dtype");
  if (M == 0 || N == 0) return ISPA_OK;
  if (!ptr_ok(A) || !ptr_ok(W) || !ptr_ok(y)) return fail(ISPA_ERR_INVALID_ARG, "pointers must be non-NULL and 16-byte aligned");
  const size_t yb = (size_t)M * N * (y_dtype == ISPA_BF16 ? 2 : 4);
  if (overlaps(y, yb, A, (size_t)M * K * 2) || overlaps(y, yb, W, (size_t)K * N * 2))
    return fail(ISPA_ERR_INVALID_ARG, "y must not overlap the inputs");
  return launch_gemm_bf16(M, N, K, A, W, y, y_dtype, (cudaStream_t)stream);
}

ispa_status ispa_gemm_q8(int M, int N, int K, const void *q, const float *sa, const void *qT, const float *sw,
                         ispa_q8_format fmt, void *y, ispa_dtype y_dtype, ispa_stream_t stream) {
  if (M < 0 || N < 0 || N % 16 != 0 || !q8_k_ok(K))
    return fail(ISPA_ERR_INVALID_ARG, "need M >= 0, N a multiple of 16 and K a positive multiple of 16");
  if (!q8_ok(fmt)) return fail(ISPA_ERR_INVALID_ARG, "bad 8-bit format");
  if (fmt == ISPA_Q8_INT8 && K > kQ8Int8MaxK) return fail(ISPA_ERR_INVALID_ARG, "int8 products need K <= 131072");
  if (!dtype_ok(y_dtype)) return fail(ISPA_ERR_INVALID_ARG, "bad y dtype");
  if (M == 0 || N == 0) return ISPA_OK;
  if (!ptr_ok(q) || !ptr_ok(sa) || !ptr_ok(qT) || !ptr_ok(sw) || !ptr_ok(y))
    return fail(ISPA_ERR_INVALID_ARG, "pointers must be non-NULL and 16-byte aligned");
  const size_t yb = (size_t)M * N * (y_dtype == ISPA_BF16 ? 2 : 4);
  if (overlaps(y, yb, q, (size_t)M * K) || overlaps(y, yb, sa, (size_t)M * 4) ||
      overlaps(y, yb, qT, (size_t)N * K) || overlaps(y, yb, sw, (size_t)N * 4))
    return fail(ISPA_ERR_INVALID_ARG, "y must not overlap the inputs");
  return launch_gemm_q8(M, N, K, q, sa, qT, sw, fmt, y, y_dtype, (cudaStream_t)stream);
}

size_t ispa_attn_local_proj_q8_workspace_bytes(const ispa_attn_desc *desc) {
  const size_t base = (ispa_attn_local_proj_workspace_bytes(desc) + 255) & ~size_t(255);
  if (base == 0) return 0;
  const size_t rows = (size_t)desc->B * ((size_t)(desc->cur_end - desc->cur_begin) * desc->tokens_per_frame);
  const size_t qa = rows * desc->H * desc->head_dim, sa = rows * 4;
  return base + ((qa + 255) & ~size_t(255)) + ((sa + 255) & ~size_t(255));
}

ispa_status ispa_attn_local_proj_q8(const ispa_attn_desc *desc, const void *q, const void *k, const void *v,
                                    const void *qT, const float *sw, ispa_q8_format fmt, int Dout, void *y,
                                    ispa_dtype y_dtype, void *workspace, size_t workspace_bytes,
                                    ispa_stream_t stream) {
  GroupRanges g;
  float scale;
  ispa_status st = attn_ranges(desc, &g, &scale);
  if (st != ISPA_OK) return st;
  if (desc->in_dtype != ISPA_BF16 || desc->head_dim != 128)
    return fail(ISPA_ERR_UNSUPPORTED, "post-switch projection is compiled for bf16 inputs with head_dim 128");
  if (!q8_ok(fmt)) return fail(ISPA_ERR_INVALID_ARG, "bad 8-bit format");
  if (fmt == ISPA_Q8_INT8 && desc->H * desc->head_dim > kQ8Int8MaxK)
    return fail(ISPA_ERR_INVALID_ARG, "int8 products need D <= 131072");
  if (Dout < 16 || Dout % 16 != 0) return fail(ISPA_ERR_INVALID_ARG, "Dout must be a positive multiple of 16");
  if (!dtype_ok(y_dtype)) return fail(ISPA_ERR_INVALID_ARG, "bad y dtype");
  if (!ptr_ok(q) || !ptr_ok(k) || (!ptr_ok(v) && desc->v_layout != ISPA_KV_E4M3_PREPARED) || !ptr_ok(qT) ||
      !ptr_ok(sw) || !ptr_ok(y))
    return fail(ISPA_ERR_INVALID_ARG, "pointers must be non-NULL and 16-byte aligned");
  const size_t need = ispa_attn_local_proj_q8_workspace_bytes(desc);
  if (!workspace || workspace_bytes < need || !aligned16(workspace))
    return fail(ISPA_ERR_INVALID_ARG, "workspace needs %zu bytes (16-byte aligned)", need);
  ispa_attn_desc d = *desc;
  d.hist_begin = d.hist_end = 0;
  d.out_dtype = ISPA_BF16;
  g.hist_begin = g.hist_end = 0;
  const int D = d.H * d.head_dim;
  const size_t rows = (size_t)d.B * g.Lq;
  const size_t a_bytes = ((rows * D * 2) + 255) & ~size_t(255);
  const size_t l_bytes = ((rows * d.H * 4) + 255) & ~size_t(255);
  const size_t base = (ispa_attn_local_proj_workspace_bytes(desc) + 255) & ~size_t(255);
  const size_t qa_bytes = (rows * D + 255) & ~size_t(255);
  char *w = static_cast<char *>(workspace);
  void *a_loc = w;
  float *lse = reinterpret_cast<float *>(w + a_bytes);
  void *attn_ws = w + a_bytes + l_bytes;
  void *qa = w + base;
  float *sa = reinterpret_cast<float *>(w + base + qa_bytes);
  cudaStream_t s = (cudaStream_t)stream;
  st = launch_attn_tc(d, g, scale, q, k, v, a_loc, lse, nullptr, nullptr, nullptr, nullptr, attn_ws, s);
  if (st != ISPA_OK) return st;
  if ((st = launch_quant_rows((int)rows, D, a_loc, fmt, qa, sa, s)) != ISPA_OK) return st;
  return launch_gemm_q8((int)rows, Dout, D, qa, sa, qT, sw, fmt, y, y_dtype, s);
}

ispa_status ispa_kv_evicted_desc(const ispa_attn_desc *desc, ispa_attn_desc *evicted) {
  GroupRanges g;
  float scale;
  ispa_status st = attn_ranges(desc, &g, &scale);
  if (st != ISPA_OK) return st;
  if (!evicted) return fail(ISPA_ERR_INVALID_ARG, "evicted is NULL");
  // kept frame f moves to its rank among the kept frames
  ispa_attn_desc e = *desc;
  const int S = desc->sink_frames, cb = desc->cur_begin, ce = desc->cur_end;
  const int rank_cb = cb < S ? cb : S;
  e.sink_frames = S;
  e.cur_begin = rank_cb;
  e.cur_end = rank_cb + (ce - cb);
  e.hist_begin = e.hist_end = 0;
  e.kv_frames = ce > S ? rank_cb + (ce - cb) : S;  // |[0, S) u [cb, ce)|
  *evicted = e;
  return ISPA_OK;
}

ispa_status ispa_kv_evict_history(const ispa_attn_desc *desc, const void *k, const void *v, void *k_out, void *v_out,
                                  ispa_stream_t stream) {
  return kv_remap(desc, k, v, k_out, v_out, true, (cudaStream_t)stream);
}

ispa_status ispa_kv_restore(const ispa_attn_desc *desc, const void *k_ev, const void *v_ev, void *k_full,
                            void *v_full, ispa_stream_t stream) {
  return kv_remap(desc, k_ev, v_ev, k_full, v_full, false, (cudaStream_t)stream);
}

ispa_status ispa_selftest_wait_timeout(long long wait_ns, ispa_stream_t stream) {
  if (wait_ns < 1000000LL || wait_ns > 10000000000LL)
    return fail(ISPA_ERR_INVALID_ARG, "wait_ns must lie in [1 ms, 10 s] (got %lld)", wait_ns);
  DevErr e;
  ispa_status st = device_err(&e);
  if (st != ISPA_OK) return st;
  e.limit_ns = wait_ns;
  return launch_selftest_wait(e, (cudaStream_t)stream);
}

ispa_status ispa_stats_reset(int D, int Dout, float *G, float *C, double *r2, ispa_stream_t stream) {
  if (D < 1 || Dout < 1) return fail(ISPA_ERR_INVALID_ARG, "D and Dout must be >= 1");
  if (!G || !C || !r2) return fail(ISPA_ERR_INVALID_ARG, "G, C and r2 must be device pointers");
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(G, 0, (size_t)D * D * sizeof(float), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(C, 0, (size_t)D * Dout * sizeof(float), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(r2, 0, sizeof(double), s);
  return cuda_status(e, "statistics reset");
}

}  // extern "C"
