"""Full-size workloads against the oracle: the 14B-shaped layer and the 30-layer
1.3B-shaped warmup + switch.

Both follow the stage-wise parity of the survey: attention on sampled query
rows x all heads x all keys; the statistics recomputed in fp64 from the GPU's
own attention rows; the solve and epsilon from the GPU's own statistics; the
selection from the oracle's epsilon.  Inputs: the drift history generator
(sink frames plus a seeded rank-64 drift and N(0, 0.1) noise per history
frame, a per-layer amplitude), fresh N(0, 1) queries and current frames per
chunk, bf16.
"""
import numpy as np
import pytest
import torch

import kv_cache_compression_two_b200 as ispa
import synth_inputs as si
from oracle import ispa_oracle as orc
from gpu_helpers import assert_lse, dev, host, max_over_rms, rel_fro

pytestmark = pytest.mark.gpu

LAMBDA_REL = 1e-4


def _eps_bound(Gs, Cs, r2, dW_ref, lam, rel_dw, stats_rel=0.0):
    """|eps - eps*| for a dW within rel_dw of the oracle's dW* (eps is the quadratic
    r2 - 2<dW, C> + <dW, G dW> and (G + lam I) dW* = C), plus 1e-6 r2 for the
    kernel's rounding and stats_rel of each term for statistics that carry an error."""
    n2 = float(np.sum(dW_ref * dW_ref))
    # |G|_2 <= the largest absolute row sum (G symmetric): an O(D^2) bound in place of an SVD
    g2 = float(np.abs(Gs).sum(axis=1).max())
    extra = 0.0
    if stats_rel > 0:
        t = abs(float(np.sum(dW_ref * Cs)))
        qd = abs(float(np.sum(dW_ref * (Gs @ dW_ref))))
        extra = stats_rel * (r2 + 2 * t + qd)
    return 1e-6 * r2 + 2.0 * lam * rel_dw * n2 + g2 * rel_dw ** 2 * n2 + extra


def _sym(G_upper):
    U = np.triu(G_upper)
    return U + np.triu(U, 1).T


class LayerCache:
    """One layer's device KV cache (bf16 K, V, prepared fp16 V) in the sink |
    history | current layout; each chunk writes its current frames."""

    def __init__(self, sh, prefix, out_dtype=ispa.ISPA_F32):
        self.sh = sh
        full = (sh.B, sh.Lkv, sh.H, sh.d)
        self.k = torch.empty(full, dtype=torch.bfloat16, device="cuda")
        self.v = torch.empty(full, dtype=torch.bfloat16, device="cuda")
        n = sh.cur_begin * sh.tpf
        self.k[:, :n] = dev(prefix["k"], torch.bfloat16)
        self.v[:, :n] = dev(prefix["v"], torch.bfloat16)
        self.desc = ispa.attn_desc(sh, ispa.ISPA_BF16, out_dtype)
        self.pdesc = ispa.prepared(self.desc)
        self.v16 = torch.empty(ispa.ispa_v16_bytes(self.desc), dtype=torch.uint8, device="cuda")
        self.first = True

    def write_chunk(self, cq):
        sh = self.sh
        rows = slice(sh.cur_begin * sh.tpf, sh.cur_end * sh.tpf)
        self.k[:, rows] = dev(cq["k"], torch.bfloat16)
        self.v[:, rows] = dev(cq["v"], torch.bfloat16)
        if self.first:  # the cache's first fill: every frame
            ispa.ispa_v16_prepare(self.desc, self.v, 0, sh.kv_frames, self.v16)
            self.first = False
        else:           # later chunks: their own frames only
            ispa.ispa_v16_prepare(self.desc, self.v, sh.cur_begin, sh.cur_end, self.v16)

    def attend(self, q):
        sh = self.sh
        o = {n: torch.empty((sh.B, sh.Lq, sh.H, sh.d), device="cuda") for n in ("loc", "full")}
        l = {n: torch.empty((sh.B, sh.Lq, sh.H), device="cuda") for n in ("loc", "full")}
        ispa.ispa_attn_split(self.pdesc, q, self.k, self.v16, o["loc"], l["loc"], None, None, o["full"], l["full"])
        return o, l


def _check_rows(sh, q_np, k_np, v_np, o, l, rows):
    ref = orc.split_attention(sh, q_np, k_np, v_np, rows=rows)
    for n in ("loc", "full"):
        got = host(o[n])[:, rows]
        err = max_over_rms(got, ref["O_" + n])
        assert err <= 1e-2, (n, err)
        assert_lse(host(l[n])[:, rows], ref["L_" + n], 1e-3)


# ---------------------------------------------------------------- 14B-shaped layer
def test_14b_layer_attention_statistics_and_solve():
    """40 heads x 128 (D = 5120), 1560 tokens per frame, sink 3 + history 60 + chunk 3
    (4680 queries over 102 960 keys, 1480 query tiles).  Attention on sampled rows x all
    heads x all keys; G, C, r2 of the first chunk against the fp64 statistics of the
    GPU's own rows; after all 8 warmup chunks (T = 37 440 rows) the full 5120 x 5120
    solve (plain and refined) against the oracle's solve of the GPU's statistics.
    (One chunk alone has fewer rows than dimensions: its G is singular, and the tf32
    statistics' rounding, about 1e-3 of G, then outweighs lambda = 1e-4 tr(G) / D on
    the null space, so G + lambda I is indefinite -- in fp64 as well.)"""
    sh = si.SHAPE_14B
    key = ("gpu", "cfg4")
    prefix = si.drift_layer_kv(sh, "bf16", 0, key)
    cq = si.chunk_qkv(sh, "bf16", 0, 0, key)
    cache = LayerCache(sh, prefix)
    cache.write_chunk(cq)
    q = dev(cq["q"], torch.bfloat16)
    o, l = cache.attend(q)
    ispa.ispa_check_device_error()
    k_np = si.assemble_kv(prefix["k"], cq["k"], sh)
    v_np = si.assemble_kv(prefix["v"], cq["v"], sh)
    del prefix
    rows = np.r_[0, 127, 128, 2339, 3071, 4608:4680:24, 4679]
    _check_rows(sh, cq["q"], k_np, v_np, o, l, rows)
    del k_np, v_np

    # statistics of the chunk, the fp64 oracle fed the GPU's own attention rows
    D, T = sh.D, sh.B * sh.Lq
    W = si.projection_weight(D, D, key)
    Wd = dev(W)
    G = torch.zeros((D, D), device="cuda")
    C = torch.zeros((D, D), device="cuda")
    r2 = torch.zeros(1, dtype=torch.float64, device="cuda")
    ws = torch.empty(ispa.ispa_accum_stats_workspace_bytes(T, D, D), dtype=torch.uint8, device="cuda")
    a_loc, a_full = o["loc"].reshape(T, D), o["full"].reshape(T, D)
    ispa.ispa_accum_stats(T, D, D, a_loc, a_full, Wd, G, C, r2, ispa.ISPA_PREC_TF32, ws)
    Gr, Cr, r2r = orc.absorption_stats(host(a_loc), host(a_full), W)
    Gh, Ch = host(G), host(C)
    iu = np.triu_indices(D)
    assert rel_fro(Gh[iu], Gr[iu]) <= 1e-3, rel_fro(Gh[iu], Gr[iu])
    assert rel_fro(Ch, Cr) <= 1e-3, rel_fro(Ch, Cr)
    assert abs(float(r2.item()) - r2r) <= 1e-3 * r2r
    del o, l, Gr, Cr, Gh, Ch
    # the other seven warmup chunks of the layer: written into the cache, attended, accumulated
    for c in range(1, 8):
        cq = si.chunk_qkv(sh, "bf16", 0, c, key)
        cache.write_chunk(cq)
        o, l = cache.attend(dev(cq["q"], torch.bfloat16))
        ispa.ispa_accum_stats(T, D, D, o["loc"].reshape(T, D), o["full"].reshape(T, D), Wd, G, C, r2,
                              ispa.ISPA_PREC_TF32, ws)
        del o, l
    ispa.ispa_check_device_error()
    del ws, cache
    Gh, Ch = host(G), host(C)

    # the 5120 x 5120 solve from the GPU's statistics of the 8 chunks (37 440 rows)
    Gs = _sym(Gh.astype(np.float32).astype(np.float64))
    Cs = Ch.astype(np.float32).astype(np.float64)
    lam32 = float(np.float32(orc.ridge_lambda(Gs, LAMBDA_REL, True)))
    ref = orc.ridge_solve(Gs, Cs, lam32)
    r2v = float(r2.item())
    rws = torch.empty(ispa.ispa_ridge_workspace_bytes(D, D), dtype=torch.uint8, device="cuda")
    for refine, tol in ((0, 1e-2), (2, 1e-5)):
        dW = torch.empty((D, D), device="cuda")
        eps = torch.zeros(1, dtype=torch.float64, device="cuda")
        ispa.ispa_ridge_solve(D, D, G, C, r2, LAMBDA_REL, True, refine, dW, eps, rws)
        ispa.ispa_check_device_error()
        err = rel_fro(host(dW), ref)
        print(f"14B solve refine={refine}: dW rel {err:.3e}")
        assert err <= tol, (refine, err)
        ref_eps = orc.eps_from_stats(Gs, Cs, r2v, ref)
        assert abs(float(eps.item()) - ref_eps) <= _eps_bound(Gs, Cs, r2v, ref, lam32, tol), (refine, eps.item(),
                                                                                              ref_eps)


# ---------------------------------------------------------------- 1.3B-shaped 30-layer model
def test_1p3b_30_layer_warmup_and_selection():
    """30 layers of the 1.3B shape, 8 warmup chunks each (T = 37 440 rows per layer),
    one solve per layer, ISPA-0.5 (K = 15).  Every layer's dW and epsilon against the
    oracle's solve of the GPU's statistics; two layers' statistics against the fp64
    statistics of their GPU rows; sampled attention rows of two layers; the selected
    set against the oracle's selection, with the epsilon gap at the K boundary
    reported against the propagated error."""
    sh = si.SHAPE_1P3B
    N, chunks, x = 30, 8, 0.5
    K = orc.num_selected(x, N)
    assert K == 15
    key = ("gpu", "cfg3")
    D, T1 = sh.D, sh.B * sh.Lq
    stats_layers = (0, 17)
    attn_checks = {(0, 0), (29, 7)}
    rws = torch.empty(ispa.ispa_ridge_workspace_bytes(D, D), dtype=torch.uint8, device="cuda")
    ws = torch.empty(ispa.ispa_accum_stats_workspace_bytes(T1, D, D), dtype=torch.uint8, device="cuda")
    eps_gpu = torch.zeros(N, dtype=torch.float64, device="cuda")
    eps_ref, dW_err, eps_dev = [], [], []
    for layer in range(N):
        prefix = si.drift_layer_kv(sh, "bf16", layer, key)
        W = si.projection_weight(D, D, key + (layer,))
        Wd = dev(W)
        cache = LayerCache(sh, prefix)
        G = torch.zeros((D, D), device="cuda")
        C = torch.zeros((D, D), device="cuda")
        r2 = torch.zeros(1, dtype=torch.float64, device="cuda")
        rows_loc, rows_full = [], []
        for c in range(chunks):
            cq = si.chunk_qkv(sh, "bf16", layer, c, key)
            cache.write_chunk(cq)
            q = dev(cq["q"], torch.bfloat16)
            o, l = cache.attend(q)
            a_loc, a_full = o["loc"].reshape(T1, D), o["full"].reshape(T1, D)
            ispa.ispa_accum_stats(T1, D, D, a_loc, a_full, Wd, G, C, r2, ispa.ISPA_PREC_TF32, ws)
            if layer in stats_layers:
                rows_loc.append(host(a_loc))
                rows_full.append(host(a_full))
            if (layer, c) in attn_checks:
                rows = np.r_[0, 1000, 2339, 4679]
                _check_rows(sh, cq["q"], si.assemble_kv(prefix["k"], cq["k"], sh),
                            si.assemble_kv(prefix["v"], cq["v"], sh), o, l, rows)
        dW = torch.empty((D, D), device="cuda")
        ispa.ispa_ridge_solve(D, D, G, C, r2, LAMBDA_REL, True, 0, dW, eps_gpu[layer:layer + 1], rws)
        ispa.ispa_check_device_error()
        Gh, Ch, r2v = host(G), host(C), float(r2.item())
        if layer in stats_layers:
            Gr, Cr, r2r = orc.absorption_stats(np.concatenate(rows_loc), np.concatenate(rows_full), W)
            iu = np.triu_indices(D)
            assert rel_fro(Gh[iu], Gr[iu]) <= 1e-3 and rel_fro(Ch, Cr) <= 1e-3, layer
            assert abs(r2v - r2r) <= 1e-3 * r2r, layer
        Gs, Cs = _sym(Gh), Ch
        lam32 = float(np.float32(orc.ridge_lambda(Gs, LAMBDA_REL, True)))
        ref = orc.ridge_solve(Gs, Cs, lam32)
        err = rel_fro(host(dW), ref)
        assert err <= 1e-2, (layer, err)
        e_ref = orc.eps_from_stats(Gs, Cs, r2v, ref)
        e_gpu = float(eps_gpu[layer].item())
        assert abs(e_gpu - e_ref) <= _eps_bound(Gs, Cs, r2v, ref, lam32, 1e-2), (layer, e_gpu, e_ref)
        eps_ref.append(e_ref)
        dW_err.append(err)
        eps_dev.append(abs(e_gpu - e_ref) / e_ref)
        del cache, G, C
    # selection: the GPU's selection on its epsilon against the oracle's on its own
    mask = torch.zeros(N, dtype=torch.uint8, device="cuda")
    idx = torch.zeros(K, dtype=torch.int32, device="cuda")
    ispa.ispa_select_layers(N, eps_gpu, K, mask, idx)
    torch.cuda.synchronize()
    _, ref_idx = orc.select_layers(eps_ref, K)
    srt = np.sort(eps_ref)
    gap = (srt[K] - srt[K - 1]) / srt[K]
    print(f"30-layer model: selected {ref_idx.tolist()}; eps range {srt[0]:.4e}..{srt[-1]:.4e}; boundary gap "
          f"{gap:.3e} vs max relative eps deviation {max(eps_dev):.3e}; max dW rel {max(dW_err):.3e}")
    if gap > 2 * max(eps_dev):
        assert idx.cpu().numpy().tolist() == ref_idx.tolist()
    else:   # a tie within the propagated error: both selections are valid, the set need not match
        pytest.skip(f"selection boundary is a tie within tolerance (gap {gap:.2e}, deviation {max(eps_dev):.2e})")
