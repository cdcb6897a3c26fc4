/*
 * ispa.h -- C ABI of the ISPA hot path on NVIDIA B200 (sm_100a).
 *
 * ISPA (Instance-Specific Parametric Absorption) compresses the KV cache of an
 * autoregressive video generator.  During a short warmup every layer runs a
 * decomposable two-group attention, accumulates absorption statistics, and at
 * the transition solves a closed-form ridge problem per layer; the K layers
 * with the smallest reconstruction error then drop their history and project
 * with W + dW.
 *
 * Passages cited below (all about arXiv 2607.00712, "Towards Memory-Efficient
 * Autoregressive Video Generation via Instance-Specific Parametric Absorption"):
 *   [EN-notes]   en.papernotes.org note, "Key Designs" 1-3 and "Loss & Training".
 *   [DE-summary] gist.science/de, "Technisches Resümee", section 2 "Methodik"
 *                ("Dual-Stream Warmup", "Layer Absorb", "Speichereffiziente
 *                Inferenz", "Dynamische Layerauswahl").
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *     allocates no memory; calls that need scratch take a caller-owned
 *     workspace whose size is given by the matching *_workspace_bytes query.
 *   - Every call validates its arguments on the host before touching the GPU
 *     and returns ISPA_ERR_INVALID_ARG / ISPA_ERR_UNSUPPORTED without launching
 *     anything.  Otherwise it enqueues kernels on `stream` and returns without
 *     synchronising (ISPA_ERR_CUDA if a launch fails).
 *   - Conditions found on the device (a non positive-definite matrix, a bounded
 *     wait that timed out) are recorded in a per-device error word and are
 *     reported by ispa_check_device_error(), which synchronises the stream.
 *   - Tensor pointers must be 16-byte aligned.  Row-major, C-contiguous layouts.
 *   - ispa_last_error() returns a thread-local description of the last failure.
 *   - Matrices act on row vectors: y = a W with W of shape [D_in, D_out].
 */
#ifndef ISPA_H
#define ISPA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t.  NULL selects the legacy default stream. */
typedef struct CUstream_st *ispa_stream_t;

typedef enum {
  ISPA_OK = 0,
  ISPA_ERR_INVALID_ARG = 1, /* bad pointer, size, range or alignment           */
  ISPA_ERR_UNSUPPORTED = 2, /* valid but not compiled (dtype / head_dim combo)  */
  ISPA_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed       */
  ISPA_ERR_NOT_SPD = 4,     /* G + lambda I had a non-positive Cholesky pivot    */
  ISPA_ERR_TIMEOUT = 5      /* a bounded device-side wait gave up                */
} ispa_status;

typedef enum { ISPA_F32 = 0, ISPA_BF16 = 1 } ispa_dtype;

/* 8-bit format of the W8A8 projection (one byte per value). */
typedef enum {
  ISPA_Q8_E4M3 = 0, /* fp8 e4m3 (bias 7, max 448), round to nearest even, saturating */
  ISPA_Q8_INT8 = 1  /* two's-complement int8 in [-127, 127], round half to even        */
} ispa_q8_format;

/* Arithmetic of the absorption-statistics GEMMs. */
typedef enum {
  ISPA_PREC_TF32 = 0, /* tcgen05 kind::tf32, operands rounded to nearest tf32, fp32 accumulate */
  ISPA_PREC_F32 = 1   /* fp32 FFMA (CUDA cores), for fp32 workloads that need fp32 accuracy   */
} ispa_precision;

/* Returns a static version string. */
const char *ispa_version(void);

/* Thread-local text of the last error reported by this thread ("" if none). */
const char *ispa_last_error(void);

/*
 * Number of kernels this library has enqueued in this process, over all
 * threads and devices (a monotonically increasing diagnostic counter; the
 * difference across a region counts the library's launches in it).
 */
uint64_t ispa_launch_count(void);

/*
 * Synchronises `stream`, then reads and clears the error word of the current
 * device.  Returns ISPA_OK, ISPA_ERR_NOT_SPD or ISPA_ERR_TIMEOUT (or
 * ISPA_ERR_CUDA if the synchronisation itself failed).  `detail` (optional,
 * host) receives the code's argument: the 1-based failing pivot for NOT_SPD,
 * the kernel's wait-site id for TIMEOUT.
 */
ispa_status ispa_check_device_error(ispa_stream_t stream, int *detail);

/*
 * Failure-detection self-test.  Launches one CTA whose thread waits, through
 * the bounded wait that every kernel of this library uses for its hand-offs,
 * on a shared-memory mbarrier that nothing ever completes, with the time limit
 * wait_ns (1 ms to 10 s).  When the limit passes it records ISPA_ERR_TIMEOUT
 * with the site ISPA_SELFTEST_SITE in the device error word — what a kernel
 * whose peer role never arrives does — and returns; nothing faults or traps,
 * so ispa_check_device_error then reports the timeout and the context stays
 * usable.  Asynchronous; ISPA_ERR_INVALID_ARG for wait_ns out of range.
 */
#define ISPA_SELFTEST_SITE 999
ispa_status ispa_selftest_wait_timeout(long long wait_ns, ispa_stream_t stream);

/* ------------------------------------------------------------------------- */
/* Two-group attention                                                        */
/* ------------------------------------------------------------------------- */
/*
 * Frame layout of one attention call.  Each instance's K/V buffer holds
 * kv_frames * tokens_per_frame token rows, frame-ordered.  The queries are the
 * current chunk: frames [cur_begin, cur_end), so Lq = (cur_end - cur_begin) *
 * tokens_per_frame.
 *   local group   = frames [0, sink_frames) united with [cur_begin, cur_end)
 *                   (a frame in both counts once);
 *   history group = frames [hist_begin, hist_end); it must not intersect the
 *                   local group.  hist_begin == hist_end means no history.
 * The local group is the sink frame(s) plus the current frame(s), the history
 * group the frames between them [EN-notes, Key Designs 1].
 * A post-switch F-layer (full context) is the same call with
 * sink_frames = cur_begin and an empty history.
 */
/* What the v argument of the attention calls points at (ispa_attn_desc.v_layout). */
typedef enum {
  ISPA_V_PLAIN = 0,       /* V in in_dtype, [B, kv_frames*tpf, H, d]; a bf16 call
                             converts the rows it reads into its workspace       */
  ISPA_V_F16_PREPARED = 1, /* a prepared fp16 copy of a bf16 V (ispa_v16_prepare) */
  ISPA_KV_E4M3_PREPARED = 2 /* k: a prepared fp8 K and V (ispa_kv8_prepare); v unused */
} ispa_v_layout;

typedef struct {
  int B;                /* independent instances (batch)                        */
  int H;                /* heads                                                */
  int head_dim;         /* d: 128 for bf16 inputs; 32, 64 or 128 for fp32       */
  int tokens_per_frame; /* tpf >= 1                                             */
  int sink_frames;      /* local part 1: frames [0, sink_frames)                */
  int hist_begin, hist_end;
  int cur_begin, cur_end;
  int kv_frames;        /* frames held per instance; row stride of K/V          */
  ispa_dtype in_dtype;  /* dtype of Q, K, V                                     */
  ispa_dtype out_dtype; /* dtype of the O outputs                               */
  float softmax_scale;  /* <= 0 selects 1/sqrt(head_dim)                        */
  ispa_v_layout v_layout; /* ISPA_V_PLAIN, ISPA_V_F16_PREPARED or ISPA_KV_E4M3_PREPARED (bf16, d = 128) */
} ispa_attn_desc;

/*
 * Decomposable dual-stream attention [EN-notes, Key Designs 1; DE-summary 2,
 * "Dual-Stream Warmup"]: the same queries attend separately to the local and
 * the history group; each group emits its normalised output O and its
 * log-sum-exp L = log sum_j exp(scale * q.k_j) (natural log, scale included).
 * With o_full/lse_full given, the kernel also merges the two groups by their
 * LSE into the full-context output (the fused form of ispa_lse_merge).
 *
 *   q          [B, Lq, H, d]                 in_dtype
 *   k, v       [B, kv_frames*tpf, H, d]      in_dtype
 *   o_loc      [B, Lq, H, d] out_dtype, lse_loc  [B, Lq, H] fp32   (required)
 *   o_hist     [B, Lq, H, d] out_dtype, lse_hist [B, Lq, H] fp32   (both or neither)
 *   o_full     [B, Lq, H, d] out_dtype, lse_full [B, Lq, H] fp32   (both or neither)
 * An empty group yields O = 0 and L = -inf.  Compiled paths: bf16 in with
 * head_dim 128 (tcgen05 tensor cores, fp32 accumulation) and fp32 in with
 * head_dim 32/64/128 (fp32 CUDA cores).  Outputs may not alias inputs.
 * Every K/V row that a group's 128-row tiles cover must hold finite values.
 *   workspace  >= ispa_attn_split_workspace_bytes(desc) bytes, 16-byte aligned
 *              (0 for fp32 inputs and for a prepared V; for bf16 inputs with
 *              v_layout ISPA_V_PLAIN it holds a power-of-two scaled fp16 copy
 *              of the V rows in use, so that the softmax weights enter the PV
 *              product with 11 significant bits).
 */
size_t ispa_attn_split_workspace_bytes(const ispa_attn_desc *desc);

ispa_status ispa_attn_split(const ispa_attn_desc *desc, const void *q, const void *k,
                            const void *v, void *o_loc, float *lse_loc, void *o_hist,
                            float *lse_hist, void *o_full, float *lse_full, void *workspace,
                            size_t workspace_bytes, ispa_stream_t stream);

/*
 * Prepared fp16 V.  The tensor-core attention multiplies the softmax weights P
 * (fp16, 11 significant bits) with an fp16 copy of V scaled by a power of two
 * per (instance, head): v16 = v * 2^e, the exact fp16 image of every bf16 value
 * whose scaled magnitude lies in [2^-14, 65504] (e = 0 unless a head's largest
 * |v| reaches 2^15 or its RMS falls below 2^-10; then e puts the largest |v| in
 * [2^14, 2^15)).  A call with v_layout ISPA_V_PLAIN converts the V rows it reads
 * on every call.  A caller that keeps V across calls -- the KV cache of a
 * generator, where a chunk writes a few new frames and the earlier ones stay --
 * keeps the converted copy instead and converts only the frames that change:
 * the history group's cost is then paid once, when its frames are written,
 * not on every chunk [EN-notes, Key Designs 1: the split attention should cost
 * no more than full attention].
 *
 * ispa_v16_bytes(desc): bytes of the prepared copy for desc's K/V layout
 *   (B * kv_frames * tpf * H * 128 fp16 values, then a per-(instance, head)
 *   state of the scale); 0 for a desc that is invalid or not bf16 with d = 128.
 * ispa_v16_prepare(desc, v, frame_begin, frame_end, v16, stream): converts the
 *   frames [frame_begin, frame_end) of every instance of the bf16 v
 *   ([B, kv_frames * tpf, H, 128]) into v16 (caller-owned, ispa_v16_bytes,
 *   16-byte aligned, not overlapping v), updating each head's state.  With
 *   frame_begin == 0 the state starts afresh: the copy then describes frames
 *   [0, frame_end), and frames past frame_end must be prepared by later calls
 *   before an attention call reads them.  When the new frames move a head's
 *   exponent, every row of that head, frames [0, kv_frames), is converted
 *   again from v, which must then hold all of them.  Asynchronous.
 * Use: set desc.v_layout = ISPA_V_F16_PREPARED and pass v16 as the v argument
 *   of ispa_attn_split, ispa_warmup_fused, ispa_attn_local_proj(_q8) (same
 *   frame layout; every row a group's 128-row tiles cover must have been
 *   prepared, from finite values).  ispa_kv_evict_history / ispa_kv_restore
 *   with that desc move a prepared copy and its state (v, v_out of their
 *   ispa_v16_bytes sizes); after a restore, prepare the history frames again as
 *   the new warmup writes them.
 */
size_t ispa_v16_bytes(const ispa_attn_desc *desc);
ispa_status ispa_v16_prepare(const ispa_attn_desc *desc, const void *v, int frame_begin, int frame_end, void *v16,
                             ispa_stream_t stream);

/*
 * Prepared fp8 K and V: attention with 8-bit products for the post-switch
 * layers.  ISPA combines with post-training 8-bit quantisation [EN-notes, Key
 * Findings (Figure 7); DE-summary 4, "Beschleunigung"]; the pages give no
 * scheme for the attention, so this library takes the plain one:
 *   * Q, K, V in fp8 e4m3 with one fp32 scale per (instance, head) over that
 *     head's rows, s = amax / 448, codes e4m3(x * (448 / amax)) (as the W8A8
 *     quantisers; Q is quantised by the attention call itself);
 *   * S = Q8 K8^T and O = P8 V8 on the 8-bit tensor cores (fp32 accumulation);
 *   * per group an online softmax over 128-key tiles taken in the group's
 *     order, each key range's tiles starting at its first key rounded down to
 *     a multiple of 16: with t = S s_q s_k scale log2(e) and a reference m
 *     per query row -- the group's first tile maximum, moved to a later tile's
 *     maximum only when that exceeds m by more than 2.75 (O and l rescaled
 *     then) -- p = 2^(t - m + 6) <= 2^8.75 (below e4m3's 448) enters the
 *     product as e4m3(p) and the normaliser l as it is (fp32); O = acc s_v / l
 *     and L = (m - 6 + log2 l) ln 2; the groups are merged by their LSE.
 * ispa_kv8_bytes(desc): bytes of the prepared buffer for desc's K/V layout
 *   (K8 [B, kv_frames*tpf, H, 128] bytes, V8 transposed [B, H, 128, rows
 *   rounded up to 16] bytes, then the per-head scales); 0 for an invalid desc
 *   or one that is not bf16 with d = 128.
 * ispa_kv8_prepare(desc, k, v, frame_begin, frame_end, kv8, stream): converts
 *   frames [frame_begin, frame_end) of the bf16 k and v into kv8 (caller-owned,
 *   16-byte aligned, not overlapping k or v).  frame_begin == 0 starts afresh
 *   (the scales then cover frames [0, frame_end)); a later prepare whose frames
 *   raise a head's amax converts every row of that head again from k / v, which
 *   must then hold all kv_frames frames.  Asynchronous.
 * Use: set desc.v_layout = ISPA_KV_E4M3_PREPARED and pass kv8 as the k argument
 *   of ispa_attn_split, ispa_attn_local_proj or ispa_attn_local_proj_q8 (v is
 *   not read and may be NULL); their workspace then holds Q's per-head amax.
 *   Not taken by ispa_warmup_fused (the warmup statistics use the bf16
 *   attention) nor by ispa_kv_evict_history / ispa_kv_restore (evict the bf16
 *   K/V, then prepare the evicted layout).
 */
size_t ispa_kv8_bytes(const ispa_attn_desc *desc);
ispa_status ispa_kv8_prepare(const ispa_attn_desc *desc, const void *k, const void *v, int frame_begin,
                             int frame_end, void *kv8, ispa_stream_t stream);

/*
 * LSE-weighted merge of two disjoint groups' results [EN-notes, Key Designs 1]:
 *   L = log(exp(L_a) + exp(L_b)),  O = exp(L_a - L) O_a + exp(L_b - L) O_b.
 * o_* [rows, H, d] (o_dtype), lse_* [rows, H] fp32, rows = B * Lq.  Both
 * groups empty (-inf) gives O = 0, L = -inf.  o_out may alias o_a or o_b
 * (element-wise in place); lse_out must not overlap lse_a or lse_b.
 * head_dim % 8 == 0.
 */
ispa_status ispa_lse_merge(int rows, int H, int head_dim, ispa_dtype o_dtype, const void *o_a,
                           const float *lse_a, const void *o_b, const float *lse_b, void *o_out,
                           float *lse_out, ispa_stream_t stream);

/* ------------------------------------------------------------------------- */
/* Absorption statistics                                                      */
/* ------------------------------------------------------------------------- */
size_t ispa_accum_stats_workspace_bytes(int T, int D, int Dout, ispa_precision prec);

/*
 * Warmup accumulation [EN-notes, Key Designs 2; DE-summary 2, "Layer Absorb"]:
 *   R = (A_full - A_loc) W,   G += A_loc^T A_loc,   C += A_loc^T R,   r2 += ||R||_F^2
 * for one batch of T activation rows taken immediately before the output
 * projection.
 *   a_loc, a_full [T, D] fp32 (D = H * head_dim, heads concatenated)
 *   W             [D, Dout] fp32
 *   G             [D, D] fp32, accumulated in place; ONLY the upper triangle
 *                 (i <= j) is written and later read, the strict lower
 *                 triangle is left as it was
 *   C             [D, Dout] fp32, accumulated in place
 *   r2            one double, accumulated in place
 *   workspace     >= ispa_accum_stats_workspace_bytes(T, D, Dout, prec) bytes
 * Zero G, C and r2 before the first batch of an instance.  T = 0 is a no-op.
 * ISPA_PREC_TF32 needs D % 32 == 0 and Dout % 32 == 0.
 */
ispa_status ispa_accum_stats(int T, int D, int Dout, const float *a_loc, const float *a_full,
                             const float *W, float *G, float *C, double *r2,
                             ispa_precision prec, void *workspace, size_t workspace_bytes,
                             ispa_stream_t stream);

/* ------------------------------------------------------------------------- */
/* Fused warmup step                                                          */
/* ------------------------------------------------------------------------- */
size_t ispa_warmup_fused_workspace_bytes(const ispa_attn_desc *desc, int Dout);

/*
 * One warmup forward step of a layer in one pass over the attention outputs
 * [EN-notes, Key Designs 1-2: the two groups' outputs come out of the same
 * attention pass, and the statistics are gathered during warmup at no extra
 * attention cost]: the two-group attention with its fused merge writes the
 * layer's full-context output O_full (fp32) and L_full, and, from the same
 * epilogue, the operands of the statistics (A_loc and A_full - A_loc rounded to
 * tf32) straight into the workspace; then G += A_loc^T A_loc (upper triangle),
 * C += A_loc^T R and r2 += ||R||^2 with R = (A_full - A_loc) W, as
 * ispa_accum_stats with ISPA_PREC_TF32 computes them from the same values.
 * The separate per-group outputs O_loc / O_hist and the statistics' rounding
 * pass over them are not materialised.
 *   desc      bf16 inputs, head_dim 128 (its out_dtype is ignored: fp32)
 *   W         [D, Dout] fp32, D = H * 128, Dout % 32 == 0
 *   o_full    [B, Lq, H, 128] fp32, l_full [B, Lq, H] fp32
 *   G, C, r2  as for ispa_accum_stats (accumulated into)
 *   workspace >= ispa_warmup_fused_workspace_bytes(desc, Dout)
 * Asynchronous; ISPA_ERR_INVALID_ARG / ISPA_ERR_UNSUPPORTED as the calls it
 * combines.
 */
ispa_status ispa_warmup_fused(const ispa_attn_desc *desc, const void *q, const void *k, const void *v,
                              const float *W, int Dout, float *o_full, float *l_full, float *G, float *C,
                              double *r2, void *workspace, size_t workspace_bytes, ispa_stream_t stream);

/* ------------------------------------------------------------------------- */
/* Closed-form absorption                                                     */
/* ------------------------------------------------------------------------- */
size_t ispa_ridge_workspace_bytes(int D, int Dout);

/*
 * Closed-form ridge solve [DE-summary 2, "Layer Absorb"; EN-notes, Key Designs 2]:
 *   dW  = (G + lambda I)^-1 C      (Cholesky LL^T = G + lambda I, dW = L^-T (L^-1 C))
 *   eps = ||A_loc (W + dW) - A_full W||_F^2 = r2 - 2<dW, C> + <dW, G dW>
 * lambda_eff = lambda, or lambda * trace(G) / D when lambda_relative != 0.
 * refine_steps extra steps of iterative refinement with fp64 residuals
 * (0 = plain fp32 solve).
 *   G [D, D] fp32 (upper triangle read), C [D, Dout] fp32, r2 one double: inputs,
 *   left unchanged.  dW [D, Dout] fp32 and eps (one double) are outputs.
 * A non-positive pivot records ISPA_ERR_NOT_SPD (see ispa_check_device_error)
 * and fills dW with NaN.  Asynchronous.
 */
ispa_status ispa_ridge_solve(int D, int Dout, const float *G, const float *C, const double *r2,
                             float lambda, int lambda_relative, int refine_steps, float *dW,
                             double *eps, void *workspace, size_t workspace_bytes,
                             ispa_stream_t stream);

/*
 * Allocation-free form of ispa_ridge_solve.  The paper has no counterpart:
 * this entry point exists for callers that cannot allocate device memory for
 * the solver's workspace -- for example a video generator's per-chunk loop
 * that must never call cudaMalloc or cudaFree (both can synchronise the whole
 * device and stall the streams that are still generating frames), or a host
 * application whose device memory is wholly owned by another allocator.
 *
 * Same arguments and results as ispa_ridge_solve, without the workspace.  Its
 * scratch is a static array inside the library sized for the largest problem
 * (2.25 ISPA_RIDGE_NOALLOC_MAX_D^2 + 64 ISPA_RIDGE_NOALLOC_MAX_D +
 * 4 ISPA_RIDGE_NOALLOC_MAX_D * ISPA_RIDGE_NOALLOC_MAX_DOUT floats, 25.25 MiB),
 * which every GPU that loads the library holds until the process exits; the call
 * itself allocates nothing.  D > ISPA_RIDGE_NOALLOC_MAX_D or Dout >
 * ISPA_RIDGE_NOALLOC_MAX_DOUT returns ISPA_ERR_INVALID_ARG, as does any size
 * whose scratch would not fit the array (checked on the host before the
 * launch).  The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) and caches it for the CUDA context that was current;
 * a call from another context (after cudaDeviceReset, for instance) looks it
 * up again.  Make the first call on a device, and the first after a reset,
 * before any stream capture.  All calls share the one array
 * and every call rewrites the parts it reads before reading them, so calls
 * that overlap on the GPU (other streams, other host threads) race: serialise
 * them.
 */
#define ISPA_RIDGE_NOALLOC_MAX_D 1024
#define ISPA_RIDGE_NOALLOC_MAX_DOUT 1024
ispa_status ispa_ridge_solve_noalloc(int D, int Dout, const float *G, const float *C, const double *r2,
                                     float lambda, int lambda_relative, int refine_steps, float *dW,
                                     double *eps, ispa_stream_t stream);

/*
 * Reconstruction error of a given correction on any statistics [EN-notes, Key
 * Designs 2 (the error), Key Designs 3 (warmup is re-entered after a scene
 * change)]: eps = r2 - 2<dW, C> + <dW, G dW> = ||A_loc (W + dW) - A_full W||_F^2
 * over the rows that G, C, r2 were accumulated from (ispa_accum_stats).  With
 * the warmup's own statistics and its solve this is the epsilon of
 * ispa_ridge_solve; with statistics gathered after the switch it is the
 * held-out error of a layer's absorption, which a caller can watch to decide
 * when to recalibrate.
 *   G [D, D] fp32 (upper triangle read), C, dW [D, Dout] fp32, r2 one double:
 *   inputs; eps one double (device): output.  fp64-accumulated reductions.
 *   workspace >= ispa_absorb_error_workspace_bytes(D, Dout).  Asynchronous.
 */
size_t ispa_absorb_error_workspace_bytes(int D, int Dout);
ispa_status ispa_absorb_error(int D, int Dout, const float *G, const float *C, const double *r2, const float *dW,
                              double *eps, void *workspace, size_t workspace_bytes, ispa_stream_t stream);

/*
 * Instance-specific layer selection [EN-notes, Key Designs 3; DE-summary 2,
 * "Dynamische Layerauswahl"]: sort the N layers by increasing eps and take
 * the K lowest as L-layers; equal eps goes to the lower layer index.
 *   eps      [N] double (device), is_local [N] uint8 (1 = L-layer),
 *   idx      [K] int32, the chosen layer indices in ascending order.
 * 0 <= K <= N <= 4096.  NaN eps sorts after every number.
 */
ispa_status ispa_select_layers(int N, const double *eps, int K, unsigned char *is_local, int *idx,
                               ispa_stream_t stream);

/*
 * W_new = W + dW for a layer that switches [DE-summary 2, "Speichereffiziente
 * Inferenz"].  W [D, Dout] in w_dtype, dW [D, Dout] fp32, W_new [D, Dout] in
 * out_dtype (rounded to nearest even).  W_new may alias W when the dtypes match.
 */
ispa_status ispa_absorb_weight(int D, int Dout, const void *W, ispa_dtype w_dtype, const float *dW,
                               void *W_new, ispa_dtype out_dtype, ispa_stream_t stream);

/* ------------------------------------------------------------------------- */
/* Post-switch layer                                                          */
/* ------------------------------------------------------------------------- */
size_t ispa_attn_local_proj_workspace_bytes(const ispa_attn_desc *desc);

/*
 * Post-switch layer step [DE-summary 2, "Speichereffiziente Inferenz";
 * EN-notes, Key Designs 3]: attention of the current chunk over the local group
 * only (the history range of desc is ignored), then the output projection
 *   y = A_loc W_proj,
 * with W_proj = W + dW for an L-layer (from ispa_absorb_weight) or the original
 * W for an F-layer (whose desc then sets sink_frames = cur_begin so that the
 * local group spans every frame).
 *   q, k, v   as for ispa_attn_split (bf16, head_dim 128)
 *   W_proj    [D, Dout] bf16,  D = H * head_dim,  Dout % 16 == 0
 *   y         [B, Lq, Dout] in y_dtype
 *   workspace >= ispa_attn_local_proj_workspace_bytes(desc) (holds A_loc in bf16
 *             and the attention workspace)
 */
ispa_status ispa_attn_local_proj(const ispa_attn_desc *desc, const void *q, const void *k,
                                 const void *v, const void *W_proj, int Dout, void *y,
                                 ispa_dtype y_dtype, void *workspace, size_t workspace_bytes,
                                 ispa_stream_t stream);

/* ------------------------------------------------------------------------- */
/* KV eviction of post-switch L-layers                                        */
/* ------------------------------------------------------------------------- */
/*
 * After the switch the selected layers drop their historical KV entries and
 * keep only the local context, sink and current frames [DE-summary 2,
 * "Speichereffiziente Inferenz"; EN-notes, Key Designs 3 and "A Worked
 * Example"].  The kept frames are the local group of desc: the union of
 * [0, sink_frames) and [cur_begin, cur_end), in frame order.
 *
 * ispa_kv_evicted_desc: the descriptor of the evicted layout, in which the
 * kept frames are stored back to back, each renumbered by its rank among the
 * kept frames: sink_frames' = sink_frames, cur_begin' = min(cur_begin,
 * sink_frames), cur_end' = cur_begin' + (cur_end - cur_begin), no history,
 * kv_frames' = the number of kept frames.  The current chunk (the queries)
 * keeps its length, and the local group of the result holds exactly the keys
 * and values of the local group of desc, in the same order, so the
 * post-switch calls (ispa_attn_split, ispa_attn_local_proj) on the evicted
 * buffers attend to the same entries.  Host only; ISPA_ERR_INVALID_ARG for an
 * invalid desc.
 *
 * ispa_kv_evict_history: copies, for every instance, the kept frames of k and
 * v (layout of desc: [B, kv_frames * tpf, H, head_dim], in_dtype) into k_out
 * and v_out (layout of the evicted desc: [B, kv_frames' * tpf, H, head_dim]),
 * bit for bit.  The caller then releases k and v: per tensor that frees
 * B * (kv_frames - kv_frames') * tpf * H * head_dim elements.  Outputs must
 * not overlap inputs; all four pointers 16-byte aligned.  Asynchronous.
 */
ispa_status ispa_kv_evicted_desc(const ispa_attn_desc *desc, ispa_attn_desc *evicted);

ispa_status ispa_kv_evict_history(const ispa_attn_desc *desc, const void *k, const void *v,
                                  void *k_out, void *v_out, ispa_stream_t stream);

/*
 * ispa_kv_restore: the inverse of ispa_kv_evict_history, for a layer that
 * goes back to full context when warmup is re-entered (recalibration below).
 * Copies the kept frames from k_ev, v_ev (layout of the evicted desc) to their
 * places in k_full, v_full (layout of desc, the descriptor the eviction used),
 * bit for bit; every other row of k_full and v_full is left as it is (the
 * history that the new warmup fills).  Same pointer rules as
 * ispa_kv_evict_history.  Asynchronous.
 */
ispa_status ispa_kv_restore(const ispa_attn_desc *desc, const void *k_ev, const void *v_ev,
                            void *k_full, void *v_full, ispa_stream_t stream);

/* ------------------------------------------------------------------------- */
/* Recalibration                                                              */
/* ------------------------------------------------------------------------- */
/*
 * Warmup can be re-entered after a major scene change, refreshing both the
 * layer selection and the weight corrections [EN-notes, Key Designs 3].  The
 * pages give no detector, so the trigger is the caller's.  Recalibration with
 * this library: for every layer ispa_stats_reset; the L-layers back to full
 * context (ispa_kv_restore into full-layout buffers, projection with W again);
 * a new warmup (ispa_attn_split, ispa_accum_stats); at its end the transition
 * as the first time (ispa_ridge_solve per layer, ispa_select_layers,
 * ispa_absorb_weight, ispa_kv_evict_history).
 *
 * ispa_stats_reset: G [D, D] and C [D, Dout] (fp32) and r2 (one double) back
 * to zero on stream, so that the next warmup accumulates from nothing.
 * Asynchronous; ISPA_ERR_INVALID_ARG for D or Dout < 1 or a NULL pointer.
 */
ispa_status ispa_stats_reset(int D, int Dout, float *G, float *C, double *r2, ispa_stream_t stream);

/* ------------------------------------------------------------------------- */
/* W8A8 post-switch projection                                                */
/* ------------------------------------------------------------------------- */
/*
 * ISPA composes with post-training W8A8 quantisation of the projections
 * [EN-notes, "Key Findings" (Figure 7); DE-summary 4, "Beschleunigung"].  The
 * pages do not fix the scheme; this library takes the plain symmetric one:
 * one scale per activation row (token) and per weight column (output
 * channel), s = amax / QMAX in fp32 (QMAX = 448 for e4m3, 127 for int8), and
 * the value q = Q(x * inv) with inv = QMAX / amax (fp32, rounded to nearest)
 * and Q the format's rounding (ispa_q8_format).  An all-zero row or column
 * gets s = 0 and q = 0.  Inputs must be finite.  The product
 *   y[m, n] = fp32(sum_k qa[m, k] qw[k, n]) * sa[m] * sw[n]
 * runs on the 8-bit tensor cores (kind::f8f6f4 for e4m3 with an fp32
 * accumulator, kind::i8 for int8 with an exact int32 one) and is rounded to
 * y_dtype at the end.
 *
 * ispa_quantize_rows: x [M, K] bf16 row-major -> q [M, K] (bytes), sa [M] fp32.
 * ispa_quantize_weight: W [K, N] bf16 row-major (the layout of W_new from
 *   ispa_absorb_weight) -> qT [N, K] (bytes, the transpose, K contiguous) and
 *   sw [N] fp32.  Once per layer, at the switch.
 * ispa_gemm_q8: y [M, N] in y_dtype from q, sa, qT, sw of the same format.
 * Sizes: M, N >= 0 with N % 16 == 0 for the product; K >= 16, K % 16 == 0;
 * for int8 products K <= 131072 (the exact int32 sum stays below 2^31).
 * Device pointers, 16-byte aligned, no overlap between inputs and outputs.
 * Asynchronous on stream; ISPA_ERR_INVALID_ARG for bad sizes, format or pointers.
 */
ispa_status ispa_quantize_rows(int M, int K, const void *x, ispa_q8_format fmt, void *q, float *sa,
                               ispa_stream_t stream);
ispa_status ispa_quantize_weight(int K, int N, const void *W, ispa_q8_format fmt, void *qT, float *sw,
                                 ispa_stream_t stream);
ispa_status ispa_gemm_q8(int M, int N, int K, const void *q, const float *sa, const void *qT,
                         const float *sw, ispa_q8_format fmt, void *y, ispa_dtype y_dtype,
                         ispa_stream_t stream);

/*
 * ispa_gemm_bf16: the bf16 projection of the post-switch layer alone,
 * y [M, N] = A [M, K] W [K, N] (A, W bf16 row-major; fp32 accumulation on the
 * tensor cores, rounded to y_dtype at the end) -- the product that W8A8
 * replaces, with the same size and pointer rules as ispa_gemm_q8.
 */
ispa_status ispa_gemm_bf16(int M, int N, int K, const void *A, const void *W, void *y, ispa_dtype y_dtype,
                           ispa_stream_t stream);

size_t ispa_attn_local_proj_q8_workspace_bytes(const ispa_attn_desc *desc);

/*
 * ispa_attn_local_proj_q8: the post-switch layer step of ispa_attn_local_proj
 * with a W8A8 projection.  The attention runs as there (A_loc in bf16); A_loc
 * is then quantised per row (ispa_quantize_rows) and multiplied with the
 * quantised weight (qT, sw from ispa_quantize_weight of W_proj, [D, Dout]).
 *   Dout % 16 == 0; y [B, Lq, Dout] in y_dtype;
 *   workspace >= ispa_attn_local_proj_q8_workspace_bytes(desc).
 */
ispa_status ispa_attn_local_proj_q8(const ispa_attn_desc *desc, const void *q, const void *k,
                                    const void *v, const void *qT, const float *sw,
                                    ispa_q8_format fmt, int Dout, void *y, ispa_dtype y_dtype,
                                    void *workspace, size_t workspace_bytes, ispa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* ISPA_H */
