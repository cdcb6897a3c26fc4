"""fp64 CPU oracle of the ISPA hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product package imports, links or
executes this module; only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may.  It is deliberately plain and slow: every
function follows the definition it cites in float64, with NumPy matmuls,
LAPACK's Cholesky and triangular solves as the only library steps, and no
blocking, fusion or reordering beyond what the definition states.

Sources (the five web pages about arXiv 2607.00712, "Towards Memory-Efficient
Autoregressive Video Generation via Instance-Specific Parametric Absorption"):

* [EN-notes]   en.papernotes.org note, section "Key Designs" 1-3, "Loss &
                Training", "Main Results" / "Ablation Study" (Table 2).
* [ZH-notes]   papernotes.org note, the Chinese version of the same sections.
* [DE-summary] gist.science/de, "Technisches Resümee", section 2 "Methodik",
                items "Dual-Stream Warmup", "Layer Absorb", "Speichereffiziente
                Inferenz" and "Dynamische Layerauswahl"; section 4, item
                "Beschleunigung" (the W8A8 combination, with the English
                note's "Key Findings").

Readings taken where the pages are silent or garbled (each one is also
listed in the design notes of the repository):

* softmax scale 1/sqrt(d); log-sum-exp in natural log with the scale included;
* no mask inside a group: the current chunk attends to itself bidirectionally;
* local group = sink frames union current frames, history = frames strictly
  between them; an empty group has L = -inf and O = 0;
* the merge (the pages cite Eq. 9-12 without printing them) is the standard
  log-sum-exp combination of two disjoint softmax groups;
* W is applied to row vectors, y = a W, W of shape [D_in, D_out];
* the ridge penalty is squared Frobenius (the DE summary writes ||.||_2^2);
* epsilon is taken over all warmup rows, without the lambda term;
* K = floor(x N); ties in epsilon go to the lower layer index;
* W8A8: symmetric per-row (activation) and per-column (weight) scales
  s = amax / QMAX in fp32, codes Q(x * QMAX / amax) in fp8 e4m3 (nearest
  even, saturating) or int8 (half to even, clamped to +-127).

Parity pins for every function live in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import math
from typing import Dict, List, Sequence, Tuple

import numpy as np
import scipy.linalg

NEG_INF = -np.inf


# ---------------------------------------------------------------------------
# attention over one KV group  [EN-notes, Key Designs 1]
# ---------------------------------------------------------------------------
def attend_group(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """Softmax attention of queries q [n, d] over one key group k, v [m, d].

    Returns the group's normalised output O [n, d] and its log-sum-exp
    L [n] = log(sum_j exp(scale * q.k_j)).  Each group yields its normalised
    value output together with the log-sum-exp of its softmax normaliser
    [EN-notes, Key Designs 1].  An empty group returns O = 0 and
    L = -inf, so that it carries no attention mass in a merge.
    """
    q = np.asarray(q, np.float64)
    n = q.shape[0]
    if k.shape[0] == 0:
        return np.zeros((n, v.shape[1])), np.full(n, NEG_INF)
    s = scale * (q @ np.asarray(k, np.float64).T)          # [n, m] scores
    m = s.max(axis=1)
    e = np.exp(s - m[:, None])
    l = e.sum(axis=1)
    O = (e @ np.asarray(v, np.float64)) / l[:, None]
    return O, m + np.log(l)


def lse_merge(o_a: np.ndarray, l_a: np.ndarray, o_b: np.ndarray, l_b: np.ndarray):
    """Recover attention over the union of two disjoint groups from each group's (O, L).

    The full output is a combination "using LSE-derived weights"; "an ordinary
    average would be incorrect because the groups generally carry different
    amounts of total attention mass" [EN-notes, Key Designs 1].  With
    L = log(exp(L_a) + exp(L_b)), O = exp(L_a - L) O_a + exp(L_b - L) O_b.
    Both groups empty gives L = -inf, O = 0.
    """
    l_a = np.asarray(l_a, np.float64)
    l_b = np.asarray(l_b, np.float64)
    L = np.logaddexp(l_a, l_b)
    both_empty = np.isneginf(L)
    Ls = np.where(both_empty, 0.0, L)
    w_a = np.where(np.isneginf(l_a), 0.0, np.exp(np.where(np.isneginf(l_a), 0.0, l_a) - Ls))
    w_b = np.where(np.isneginf(l_b), 0.0, np.exp(np.where(np.isneginf(l_b), 0.0, l_b) - Ls))
    O = w_a[..., None] * np.asarray(o_a, np.float64) + w_b[..., None] * np.asarray(o_b, np.float64)
    return O, L


def _local_rows(shape) -> np.ndarray:
    frames = sorted(set(range(0, shape.sink_frames)) | set(range(shape.cur_begin, shape.cur_end)))
    return np.array([r for f in frames for r in range(f * shape.tpf, (f + 1) * shape.tpf)], dtype=np.int64)


def _hist_rows(shape) -> np.ndarray:
    return np.arange(shape.hist_begin * shape.tpf, shape.hist_end * shape.tpf, dtype=np.int64)


def split_attention(shape, q, k, v, scale: float = None, rows: Sequence[int] = None,
                    row_block: int = 512) -> Dict[str, np.ndarray]:
    """Decomposable two-group attention of one chunk  [EN-notes, Key Designs 1; DE-summary 2].

    q [B, Lq, H, d]; k, v [B, kv_frames*tpf, H, d].  The same queries attend
    separately to the local group (sink frames and current frames) and to the
    history group (the frames in between); the two results are merged by their
    LSE into the full-context output.  ``rows`` restricts the query rows (all by
    default).  Returns O_* [B, n, H, d] and L_* [B, n, H] for loc, hist, full.
    """
    d = q.shape[-1]
    scale = 1.0 / math.sqrt(d) if not scale else scale
    B, Lq, H, _ = q.shape
    rows = np.arange(Lq) if rows is None else np.asarray(rows)
    n = len(rows)
    loc_idx, hist_idx = _local_rows(shape), _hist_rows(shape)
    out = {key: np.zeros((B, n, H, d)) for key in ("O_loc", "O_hist", "O_full")}
    out.update({key: np.zeros((B, n, H)) for key in ("L_loc", "L_hist", "L_full")})
    for b in range(B):
        for h in range(H):
            kl, vl = k[b, loc_idx, h, :], v[b, loc_idx, h, :]
            kh, vh = k[b, hist_idx, h, :], v[b, hist_idx, h, :]
            for r0 in range(0, n, row_block):
                rr = rows[r0:r0 + row_block]
                qq = np.asarray(q[b, rr, h, :], np.float64)
                o_l, l_l = attend_group(qq, kl, vl, scale)
                o_h, l_h = attend_group(qq, kh, vh, scale)
                o_f, l_f = lse_merge(o_l, l_l, o_h, l_h)
                sl = slice(r0, r0 + len(rr))
                out["O_loc"][b, sl, h], out["L_loc"][b, sl, h] = o_l, l_l
                out["O_hist"][b, sl, h], out["L_hist"][b, sl, h] = o_h, l_h
                out["O_full"][b, sl, h], out["L_full"][b, sl, h] = o_f, l_f
    return out


def full_attention(shape, q, k, v, scale: float = None, rows: Sequence[int] = None,
                   row_block: int = 512) -> Tuple[np.ndarray, np.ndarray]:
    """Monolithic softmax attention over every KV frame (the F-layer path after the switch).

    F-layers keep attending over the full context after the switch [EN-notes,
    Key Designs 3; DE-summary 2, "Speichereffiziente Inferenz"].
    """
    d = q.shape[-1]
    scale = 1.0 / math.sqrt(d) if not scale else scale
    B, Lq, H, _ = q.shape
    rows = np.arange(Lq) if rows is None else np.asarray(rows)
    n = len(rows)
    O = np.zeros((B, n, H, d))
    L = np.zeros((B, n, H))
    for b in range(B):
        for h in range(H):
            for r0 in range(0, n, row_block):
                rr = rows[r0:r0 + row_block]
                o, l = attend_group(q[b, rr, h, :], k[b, :, h, :], v[b, :, h, :], scale)
                O[b, r0:r0 + len(rr), h], L[b, r0:r0 + len(rr), h] = o, l
    return O, L


def heads_to_rows(O: np.ndarray) -> np.ndarray:
    """[B, n, H, d] -> [B*n, H*d]: one activation row per query token, heads concatenated."""
    B, n, H, d = O.shape
    return np.asarray(O, np.float64).reshape(B * n, H * d)


# ---------------------------------------------------------------------------
# absorption statistics and the closed-form solve
# [EN-notes, Key Designs 2; DE-summary 2, "Layer Absorb"]
# ---------------------------------------------------------------------------
def residual(A_loc: np.ndarray, A_full: np.ndarray, W: np.ndarray) -> np.ndarray:
    """Projected output residual R = (A_full - A_loc) W, taken before the output projection."""
    return (np.asarray(A_full, np.float64) - np.asarray(A_loc, np.float64)) @ np.asarray(W, np.float64)


def absorption_stats(A_loc: np.ndarray, A_full: np.ndarray, W: np.ndarray):
    """Sufficient statistics of the warmup rows: G = A_loc^T A_loc, C = A_loc^T R, r2 = ||R||_F^2.

    The pages accumulate "activation outer products and activation-residual
    cross-statistics" during the forward passes [EN-notes, Key Designs 2]; the
    DE summary's closed form uses exactly G and C.
    """
    A = np.asarray(A_loc, np.float64)
    R = residual(A, A_full, W)
    return A.T @ A, A.T @ R, float(np.sum(R * R))


def ridge_lambda(G: np.ndarray, lam: float, relative: bool) -> float:
    """lambda as given, or lam * tr(G) / D when ``relative``."""
    return float(lam) * float(np.trace(G)) / G.shape[0] if relative else float(lam)


def cholesky_lower(A: np.ndarray) -> np.ndarray:
    """Lower Cholesky factor of a symmetric positive-definite matrix (LAPACK potrf)."""
    return np.linalg.cholesky(np.asarray(A, np.float64))


def ridge_solve(G: np.ndarray, C: np.ndarray, lam: float) -> np.ndarray:
    """Delta W = (G + lambda I)^-1 C  [DE-summary 2, "Layer Absorb"].

    The minimiser of ||A_loc (W + dW) - A_full W||^2 + lambda ||dW||^2 is
    dW = (A_loc^T A_loc + lambda I)^-1 A_loc^T (A_full - A_loc) W.  The "single
    D x D matrix inversion" [EN-notes, Key Designs 2] is applied as a Cholesky
    factorisation LL^T = G + lambda I and two triangular solves.
    """
    G = np.asarray(G, np.float64)
    M = G + lam * np.eye(G.shape[0])
    Lf = cholesky_lower(M)
    Y = scipy.linalg.solve_triangular(Lf, np.asarray(C, np.float64), lower=True)
    return scipy.linalg.solve_triangular(Lf.T, Y, lower=False)


def eps_direct(A_loc: np.ndarray, A_full: np.ndarray, W: np.ndarray, dW: np.ndarray) -> float:
    """epsilon = ||A_loc (W + dW) - A_full W||_F^2 over all warmup rows [EN-notes, Key Designs 2]."""
    A = np.asarray(A_loc, np.float64)
    W = np.asarray(W, np.float64)
    E = A @ (W + np.asarray(dW, np.float64)) - np.asarray(A_full, np.float64) @ W
    return float(np.sum(E * E))


def eps_from_stats(G: np.ndarray, C: np.ndarray, r2: float, dW: np.ndarray) -> float:
    """The same epsilon expanded over the statistics: r2 - 2<dW, C> + <dW, G dW>.

    ||A dW - R||^2 = ||R||^2 - 2 tr(dW^T A^T R) + tr(dW^T A^T A dW).
    """
    dW = np.asarray(dW, np.float64)
    return float(r2 - 2.0 * np.sum(dW * C) + np.sum(dW * (np.asarray(G, np.float64) @ dW)))


# ---------------------------------------------------------------------------
# layer selection  [EN-notes, Key Designs 3; DE-summary 2, "Dynamische Layerauswahl"]
# ---------------------------------------------------------------------------
def num_selected(x: float, N: int) -> int:
    """ISPA-x converts K = x N layers; read as floor(x N), never above the budget."""
    return int(math.floor(x * N + 1e-9))


def select_layers(eps: Sequence[float], K: int):
    """Sort layers by increasing epsilon and take the K lowest as L-layers.

    Ties go to the lower layer index (stable sort).  A NaN epsilon (a layer
    whose solve failed) orders after every number, NaNs among themselves by
    layer index.  Returns (is_local uint8 [N], idx int32 [K] ascending by layer
    index).
    """
    eps = np.asarray(eps, np.float64)
    N = eps.shape[0]
    nan = np.isnan(eps)
    order = sorted(range(N), key=lambda i: (bool(nan[i]), 0.0 if nan[i] else float(eps[i]), i))
    chosen = sorted(order[:K])
    is_local = np.zeros(N, np.uint8)
    is_local[chosen] = 1
    return is_local, np.array(chosen, np.int32)


def kv_retained_fraction(x: float, hist_frac: float) -> float:
    """KV kept relative to full caching when a fraction x of layers drops its history.

    An L-layer keeps sink + current entries and evicts history; F-layers keep
    everything [EN-notes, Key Designs 3].  With h = history / all KV entries of a
    layer, the kept fraction is (1 - x) + x (1 - h) = 1 - x h.
    """
    return 1.0 - x * hist_frac


# ---------------------------------------------------------------------------
# post-switch L-layer  [DE-summary 2, "Speichereffiziente Inferenz"]
# ---------------------------------------------------------------------------
def evict_history(shape, kv: np.ndarray) -> np.ndarray:
    """K or V of an L-layer once its historical entries are evicted: for every
    instance, the frames of the local group (sink and current, in frame order)
    back to back.  The selected layers drop K_hist, V_hist and run on the local
    context alone [DE-summary 2, "Speichereffiziente Inferenz"; EN-notes, Key
    Designs 3 and "A Worked Example"].  kv [B, kv_frames * tpf, H, d].
    """
    return np.ascontiguousarray(np.asarray(kv)[:, _local_rows(shape)])


def restore_history(shape, kv_evicted: np.ndarray, kv_full: np.ndarray) -> np.ndarray:
    """The kept frames of an evicted buffer put back at their places in a
    full-layout buffer (every other row of ``kv_full`` unchanged), for a layer
    that returns to full context when warmup is re-entered [EN-notes, Key
    Designs 3].  kv_evicted [B, kept * tpf, H, d], kv_full [B, kv_frames * tpf, H, d].
    """
    out = np.array(kv_full, copy=True)
    out[:, _local_rows(shape)] = kv_evicted
    return out


def evicted_shape(shape):
    """Frame layout of an evicted buffer: every kept frame is renumbered by its
    rank among the kept frames, so the sink stays [0, sink), the current chunk
    keeps its length and starts at the number of kept frames before it, and
    there is no history.  Its local group holds the same keys, in the same
    order, as the local group of ``shape``, and its queries are the same.
    """
    import dataclasses
    kept = sorted(set(range(shape.sink_frames)) | set(range(shape.cur_begin, shape.cur_end)))
    rank = {f: i for i, f in enumerate(kept)}
    cb = rank[shape.cur_begin]
    return dataclasses.replace(shape, hist_begin=0, hist_end=0, cur_begin=cb,
                               cur_end=cb + shape.cur_end - shape.cur_begin, kv_frames=len(kept))


def local_projection(shape, q, k, v, W: np.ndarray, dW: np.ndarray = None, scale: float = None,
                     rows: Sequence[int] = None) -> np.ndarray:
    """Y = A_loc (W + dW): attention over sink + current only, projected with W_new = W + dW.

    Returns Y [B, n, D_out].
    """
    d = q.shape[-1]
    scale = 1.0 / math.sqrt(d) if not scale else scale
    B, Lq, H, _ = q.shape
    rows = np.arange(Lq) if rows is None else np.asarray(rows)
    loc_idx = _local_rows(shape)
    O = np.zeros((B, len(rows), H, d))
    for b in range(B):
        for h in range(H):
            O[b, :, h], _ = attend_group(q[b, rows, h, :], k[b, loc_idx, h, :], v[b, loc_idx, h, :], scale)
    Weff = np.asarray(W, np.float64) + (0.0 if dW is None else np.asarray(dW, np.float64))
    return (heads_to_rows(O) @ Weff).reshape(B, len(rows), -1)


# ---------------------------------------------------------------------------
# one layer's warmup -> transition, and a whole model's selection
# ---------------------------------------------------------------------------
def absorb_layer(chunks: List[Dict[str, np.ndarray]], W: np.ndarray, lam: float, lam_relative: bool):
    """Warmup over chunks of one layer, then its closed-form absorption.

    ``chunks`` holds the split-attention outputs of every warmup chunk (dicts
    from :func:`split_attention`).  Rows of all chunks are stacked (the
    statistics are summed over the warmup's forward calls).  Returns G, C, r2,
    lambda, dW, eps (direct form) and the stacked rows.
    """
    A_loc = np.concatenate([heads_to_rows(c["O_loc"]) for c in chunks], axis=0)
    A_full = np.concatenate([heads_to_rows(c["O_full"]) for c in chunks], axis=0)
    G, C, r2 = absorption_stats(A_loc, A_full, W)
    lam_eff = ridge_lambda(G, lam, lam_relative)
    dW = ridge_solve(G, C, lam_eff)
    return dict(G=G, C=C, r2=r2, lam=lam_eff, dW=dW, eps=eps_direct(A_loc, A_full, W, dW),
                A_loc=A_loc, A_full=A_full)


def attention_flops(n_query: int, n_key: int, H: int, d: int) -> float:
    """Dot-product FLOPs of one attention call: QK^T and PV, 2 flops per multiply-add."""
    return 4.0 * n_query * n_key * H * d


# ---------------------------------------------------------------------------
# W8A8 post-switch projection  [EN-notes, "Key Findings" (Figure 7);
# DE-summary §4 "Beschleunigung"]
# ---------------------------------------------------------------------------
# The pages report ISPA combined with W8A8 post-training quantisation but do not
# fix the scheme.  Reading taken: symmetric quantisation with one fp32 scale per
# activation row and per weight column, s = amax / QMAX, q = Q(x * inv) with
# inv = QMAX / amax; Q rounds to fp8 e4m3 (to nearest even, saturating at 448)
# or to int8 (half to even, clamped to +-127).  The scale arithmetic is fp32,
# the precision that decides the codes on both sides.
Q8_E4M3, Q8_INT8 = 0, 1
Q8_MAX = {Q8_E4M3: 448.0, Q8_INT8: 127.0}


def e4m3_round(x: np.ndarray) -> np.ndarray:
    """Nearest fp8 e4m3 value of each x (ties to even mantissa), saturating at +-448.

    The format (OCP 8-bit floating point, E4M3): sign, 4 exponent bits with bias
    7, 3 mantissa bits; normal values (1 + m/8) 2^(e-7) for e = 1..15 except
    e = 15, m = 7 (NaN), subnormals m 2^-9; no infinities.  In the binade
    [2^E, 2^(E+1)) with E >= -6 the spacing is 2^(E-3); below 2^-6 it is 2^-9.
    """
    x = np.asarray(x, np.float64)
    a = np.abs(x)
    _, ex = np.frexp(a)                      # a = f 2^ex, f in [0.5, 1)
    E = np.maximum(ex - 1, -6)               # binade exponent, floored at the normal minimum
    quantum = np.ldexp(1.0, E - 3)
    q = np.rint(a / quantum) * quantum       # exact: a / quantum is a power-of-two scaling
    q = np.minimum(q, 448.0)
    return np.copysign(q, x)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Value of each e4m3 byte (NaN for the codes S.1111.111), from the format definition."""
    c = np.asarray(codes, np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, np.ldexp(m.astype(np.float64), -9),
                   np.ldexp(1.0 + m / 8.0, e - 7))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return s * val


def q8_round(t: np.ndarray, fmt: int) -> np.ndarray:
    """The format's rounding Q of already-scaled values t."""
    if fmt == Q8_E4M3:
        return e4m3_round(t)
    return np.clip(np.rint(np.asarray(t, np.float64)), -127.0, 127.0)


def quantize_rows(x: np.ndarray, fmt: int):
    """Per-row quantisation of x [M, K]: returns (q [M, K] as float64 values, s [M] fp32).

    amax, inv = QMAX / amax and x * inv are fp32 operations (each rounded to
    nearest); an all-zero row has s = 0, inv = 0, q = 0.
    """
    x32 = np.asarray(x, np.float32)
    qmax = np.float32(Q8_MAX[fmt])
    amax = np.abs(x32).max(axis=1) if x32.shape[1] else np.zeros(x32.shape[0], np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(amax > 0, qmax / np.where(amax > 0, amax, np.float32(1)), np.float32(0)).astype(np.float32)
    s = (amax / qmax).astype(np.float32)
    t = (x32 * inv[:, None]).astype(np.float32)
    return q8_round(t.astype(np.float64), fmt), s


def quantize_cols(W: np.ndarray, fmt: int):
    """Per-column quantisation of W [K, N]: (q [K, N] values, s [N] fp32)."""
    q, s = quantize_rows(np.asarray(W, np.float32).T, fmt)
    return q.T, s


def gemm_q8(qa: np.ndarray, sa: np.ndarray, qw: np.ndarray, sw: np.ndarray, fmt: int) -> np.ndarray:
    """y[m, n] = (sum_k qa[m, k] qw[k, n]) sa[m] sw[n].

    The sum is exact in float64 for both formats (e4m3 products carry at most 8
    significant bits over a 36-bit range, int8 ones are integers below 2^15).
    For int8 the kernel's accumulator is that exact integer, and the scaling is
    taken as the kernel takes it: fp32(acc) * sa, then * sw, each in fp32 with
    rounding to nearest -- returned as fp32.  For e4m3 the exact value is
    returned in float64 (the tensor cores add in fp32).
    """
    acc = np.asarray(qa, np.float64) @ np.asarray(qw, np.float64)
    if fmt == Q8_INT8:
        a32 = acc.astype(np.float32)           # |acc| < 2^31, rounded to nearest fp32
        return (a32 * np.asarray(sa, np.float32)[:, None]).astype(np.float32) * np.asarray(sw, np.float32)[None, :]
    return acc * np.asarray(sa, np.float64)[:, None] * np.asarray(sw, np.float64)[None, :]


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Nearest bfloat16 value (8 significand bits, fp32's exponent range), ties to even.

    Written from the format: x is first rounded to fp32, then the low 16 bits of
    its encoding are rounded away (adding 0x7FFF plus the kept part's lowest bit
    carries into the kept bits exactly when the dropped part exceeds half, or
    equals half with an odd kept part).  Inputs must be finite.
    """
    b = np.ascontiguousarray(np.asarray(x, np.float32)).view(np.uint32).astype(np.uint64)
    b = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16
    return b.astype(np.uint32).view(np.float32).astype(np.float64)


def local_projection_q8(shape, q, k, v, W_new: np.ndarray, fmt: int, scale: float = None) -> np.ndarray:
    """The post-switch step with a W8A8 projection: Y [B, n, D_out].

    A_loc from the local-group attention (as in :func:`local_projection`), held
    in bf16 as the post-switch layer stores it, quantised per row; W_new
    quantised per column; the 8-bit product scaled back (:func:`gemm_q8`).
    """
    B, Lq = q.shape[0], q.shape[1]
    A = local_projection(shape, q, k, v, np.eye(shape.H * shape.d), None, scale)
    A = bf16_round(A.reshape(B * Lq, -1))
    qa, sa = quantize_rows(A, fmt)
    qw, sw = quantize_cols(W_new, fmt)
    return np.asarray(gemm_q8(qa, sa, qw, sw, fmt)).reshape(B, Lq, -1)


# ---------------------------------------------------------------------------
# FP8 post-switch attention: the W8A8 combination carried into the attention
# products (QK^T and PV in fp8 e4m3).  The pages report ISPA combined with
# post-training 8-bit quantisation [EN-notes, Key Findings (Figure 7);
# DE-summary 4, "Beschleunigung"] and give no scheme for the attention.
# Reading taken:
#  * Q, K, V: one fp32 scale per (instance, head) over that head's rows,
#    s = amax / 448, codes e4m3(x * (448 / amax)) -- the row quantiser above
#    applied to the head's values as one row;
#  * scores in log2 units t = (q8 . k8) s_q s_k scale log2(e);
#  * each group is taken in blocks of 128 keys in its order (the local group's
#    sink range, then its current range; the history range), the blocks of a
#    range starting at the 16-aligned key position at or below its first key;
#  * a reference m per query row: the first block's maximum, then moved to a
#    block's maximum only when that maximum exceeds m by more than TAU = 2.75
#    (log2 units; the product and the sum are scaled by 2^(m_old - m_new) when
#    it moves); per block p = 2^(t - m + 6), so that p <= 2^8.75 < 448 (e4m3's
#    largest finite value) and the weights of the bulk of the keys lie in
#    e4m3's normal range; the sum l += p is kept exactly, the product
#    acc += e4m3(p) v8;
#  * O = acc s_v / l, L = (m - 6 + log2 l) ln 2; the two groups are merged by
#    their log-sum-exp as in lse_merge.
# With the weights kept exact the result is softmax attention whatever m is;
# the reference only decides where each weight falls on the e4m3 grid.  A
# reference that follows the running maximum at every block (TAU = 0) needs an
# offset of at most log2(448) and rescales O whenever any row's maximum grows,
# which on long histories is most blocks; with TAU the reference settles after
# the first blocks.
# ---------------------------------------------------------------------------
FP8_BLOCK, FP8_ALIGN, FP8_P_OFFSET, FP8_TAU = 128, 16, 6.0, 2.75


def quantize_heads(x: np.ndarray):
    """Per (instance, head) e4m3 quantisation of x [B, n, H, d].

    Returns (codes as float64 values [B, n, H, d], s [B, H] fp32); each head's
    n x d values are quantised as one row by :func:`quantize_rows`.
    """
    B, n, H, d = x.shape
    q = np.empty(x.shape)
    s = np.empty((B, H), np.float32)
    for b in range(B):
        for h in range(H):
            qq, ss = quantize_rows(np.asarray(x[b, :, h, :], np.float32).reshape(1, n * d), Q8_E4M3)
            q[b, :, h, :] = qq.reshape(n, d)
            s[b, h] = ss[0]
    return q, s


def _runs(rows: np.ndarray):
    """Contiguous [lo, hi) runs of a sorted index array."""
    out = []
    for r in rows:
        if out and out[-1][1] == r:
            out[-1][1] = r + 1
        else:
            out.append([int(r), int(r) + 1])
    return [tuple(x) for x in out]


def fp8_blocks(ranges) -> List[Tuple[int, int]]:
    """The blocks of a group: for each key range [lo, hi) in order, windows of
    FP8_BLOCK keys starting at lo rounded down to FP8_ALIGN; each block is
    returned as the [first, end) of its keys that belong to the range."""
    out = []
    for lo, hi in ranges:
        w = lo - lo % FP8_ALIGN
        while w < hi:
            out.append((max(w, lo), min(w + FP8_BLOCK, hi)))
            w += FP8_BLOCK
    return out


def attend_group_fp8(t: np.ndarray, v8: np.ndarray, blocks, quantize_p: bool = True, tie_rel: float = 0.0):
    """Blockwise softmax of one group with e4m3 weights (see the reading above).

    t [n, Lkv] scores in log2 units (columns outside the group unused), v8
    [Lkv, d] dequantisation-free e4m3 codes of V, blocks from :func:`fp8_blocks`.
    Returns (acc / l [n, d] before the V scale, L in natural log [n]).
    quantize_p=False keeps the weights exact (the plain online softmax).

    With tie_rel > 0 a third array [n, d] is returned: for the weights that lie
    within a relative tie_rel of a rounding boundary of the e4m3 grid -- where a
    weight computed in another precision may round to the neighbouring code --
    the sum of (code step) |v8| / l, the most the output can move by those
    roundings; +inf for a row where a block maximum lies within tie_rel of the
    threshold that moves the reference (there the reference itself is a tie).
    """
    n, d = t.shape[0], v8.shape[1]
    if not blocks:
        empty = (np.zeros((n, d)), np.full(n, NEG_INF))
        return empty + (np.zeros((n, d)),) if tie_rel > 0 else empty
    m = None
    l = np.zeros(n)
    acc = np.zeros((n, d))
    amb = np.zeros((n, d))
    undecided = np.zeros(n, bool)
    for lo, hi in blocks:
        tb = t[:, lo:hi]
        bm = tb.max(axis=1)
        if m is None:
            m = bm
        else:
            if tie_rel > 0:  # the decision itself is a tie: any output of the row is admissible
                undecided |= np.abs(bm - (m + FP8_TAU)) <= tie_rel * np.maximum(1.0, np.abs(bm))
            m_new = np.where(bm > m + FP8_TAU, bm, m)
            f = np.exp2(m - m_new)
            acc *= f[:, None]
            amb *= f[:, None]
            l *= f
            m = m_new
        p = np.exp2(tb - m[:, None] + FP8_P_OFFSET)
        l += p.sum(axis=1)
        acc += (e4m3_round(p) if quantize_p else p) @ v8[lo:hi]
        if tie_rel > 0:
            step = np.abs(e4m3_round(p * (1.0 + tie_rel)) - e4m3_round(p * (1.0 - tie_rel)))
            amb += step @ np.abs(v8[lo:hi])
    out = (acc / l[:, None], (m - FP8_P_OFFSET + np.log2(l)) * math.log(2.0))
    if tie_rel <= 0:
        return out
    amb = amb / l[:, None]
    amb[undecided] = np.inf
    return out + (amb,)


def split_attention_fp8(shape, q, k, v, scale: float = None, rows: Sequence[int] = None,
                        quantize_p: bool = True, tie_rel: float = 0.0) -> Dict[str, np.ndarray]:
    """Two-group attention with fp8 e4m3 products (reading above); same outputs
    as :func:`split_attention`.  q, k, v hold the unquantised (bf16) values; the
    per-head quantisation is part of the definition.  With tie_rel > 0 the
    outputs also hold A_loc, A_hist, A_full [B, n, H, d]: how far each output may
    move by weights that sit within tie_rel of an e4m3 rounding boundary (see
    attend_group_fp8), after the V scale (A_full by the merge weights)."""
    d = q.shape[-1]
    scale = 1.0 / math.sqrt(d) if not scale else scale
    B, Lq, H, _ = q.shape
    rows = np.arange(Lq) if rows is None else np.asarray(rows)
    n = len(rows)
    q8, sq = quantize_heads(q)
    k8, sk = quantize_heads(k)
    v8, sv = quantize_heads(v)
    blk_loc = fp8_blocks(_runs(_local_rows(shape)))
    blk_hist = fp8_blocks(_runs(_hist_rows(shape)))
    out = {key: np.zeros((B, n, H, d)) for key in ("O_loc", "O_hist", "O_full")}
    out.update({key: np.zeros((B, n, H)) for key in ("L_loc", "L_hist", "L_full")})
    if tie_rel > 0:
        out.update({key: np.zeros((B, n, H, d)) for key in ("A_loc", "A_hist", "A_full")})
    log2e = 1.0 / math.log(2.0)
    for b in range(B):
        for h in range(H):
            c = float(sq[b, h]) * float(sk[b, h]) * scale * log2e
            t = (q8[b, rows, h, :] @ k8[b, :, h, :].T) * c          # [n, Lkv]
            res = {}
            for name, blk in (("loc", blk_loc), ("hist", blk_hist)):
                r = attend_group_fp8(t, v8[b, :, h, :], blk, quantize_p, tie_rel)
                res[name] = (r[0] * float(sv[b, h]), r[1])
                if tie_rel > 0:
                    out["A_" + name][b, :, h] = r[2] * float(sv[b, h])
            o_f, l_f = lse_merge(res["loc"][0], res["loc"][1], res["hist"][0], res["hist"][1])
            for name in ("loc", "hist"):
                out["O_" + name][b, :, h], out["L_" + name][b, :, h] = res[name]
            out["O_full"][b, :, h], out["L_full"][b, :, h] = o_f, l_f
            if tie_rel > 0:  # the merge weighs the allowances like the outputs
                out["A_full"][b, :, h] = lse_merge(out["A_loc"][b, :, h], res["loc"][1],
                                                   out["A_hist"][b, :, h], res["hist"][1])[0]
    return out
