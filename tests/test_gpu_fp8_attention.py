"""GPU parity of the fp8 e4m3 attention (prepared K/V, kind::f8f6f4) against the
oracle's fp8 attention (per-head e4m3 scales, blockwise online softmax with
e4m3 weights), and its distance from the exact attention of the bf16 inputs.

Tolerance: the oracle follows the same definition in fp64, so the kernel
differs from it by fp32 arithmetic (scores, exponentials, sums) -- max |dO| <=
1e-2 of each head's output RMS, as for the bf16 path, and LSE within 1e-3 --
and by the weights that sit so close to a rounding boundary of the e4m3 grid
that fp32 may round them to the neighbouring code.  The oracle reports how far
those can move each output (split_attention_fp8's A_* at TIE_REL) and the bound
adds it.  TIE_REL: the kernel forms p = 2^x with x = t - m + 6 in fp32 from
scores accumulated in fp32 over 128 products; for |t| up to ~32 (log2 units)
their error stays below 2^-19 |t|, so p is within a relative 2^-14 of the
exact weight."""
import dataclasses

import numpy as np
import pytest
import torch

import kv_cache_compression_two_b200 as ispa
import synth_inputs as si
from oracle import ispa_oracle as orc
from gpu_helpers import assert_lse, dev, host, nan_like, rel_fro

pytestmark = pytest.mark.gpu

SHAPES = [
    # several query tiles with a ragged tail, two local ranges, frames of 50 keys (ranges start off the 16-key grid)
    si.AttnShape(B=2, H=2, d=128, tpf=50, sink_frames=2, hist_begin=2, hist_end=7, cur_begin=7, cur_end=10,
                 kv_frames=10),
    # no history
    si.AttnShape(B=1, H=3, d=128, tpf=37, sink_frames=1, hist_begin=1, hist_end=1, cur_begin=1, cur_end=5,
                 kv_frames=5),
    # first chunk: sink = current
    si.AttnShape(B=1, H=1, d=128, tpf=200, sink_frames=2, hist_begin=2, hist_end=2, cur_begin=0, cur_end=2,
                 kv_frames=2),
    # exact multiples of the tiles, long history
    si.AttnShape(B=1, H=2, d=128, tpf=128, sink_frames=1, hist_begin=1, hist_end=9, cur_begin=9, cur_end=10,
                 kv_frames=10),
    # single-token frames
    si.AttnShape(B=3, H=1, d=128, tpf=1, sink_frames=1, hist_begin=1, hist_end=40, cur_begin=40, cur_end=43,
                 kv_frames=43),
]


def run_fp8(sh, data, out_dt=ispa.ISPA_F32, prepare=None):
    tout = torch.float32 if out_dt == ispa.ISPA_F32 else torch.bfloat16
    q, k, v = (dev(data[n], torch.bfloat16) for n in ("q", "k", "v"))
    desc = ispa.attn_desc(sh, ispa.ISPA_BF16, out_dt)
    pd = ispa.prepared(desc, ispa.ISPA_KV_E4M3_PREPARED)
    kv8 = torch.empty(ispa.ispa_kv8_bytes(desc), dtype=torch.uint8, device="cuda")
    if prepare is None:
        ispa.ispa_kv8_prepare(desc, k, v, 0, sh.kv_frames, kv8)
    else:
        prepare(desc, k, v, kv8)
    B, Lq, H = sh.B, sh.Lq, sh.H
    o = {n: nan_like((B, Lq, H, 128), tout) for n in ("loc", "hist", "full")}
    l = {n: nan_like((B, Lq, H), torch.float32) for n in ("loc", "hist", "full")}
    ws = torch.empty(ispa.ispa_attn_split_workspace_bytes(pd), dtype=torch.uint8, device="cuda")
    ispa.ispa_attn_split(pd, q, kv8, None, o["loc"], l["loc"], o["hist"], l["hist"], o["full"], l["full"],
                         workspace=ws)
    ispa.ispa_check_device_error()
    torch.cuda.synchronize()
    return {n: host(t) for n, t in o.items()}, {n: host(t) for n, t in l.items()}


TIE_REL = 2.0 ** -14


def check_against_oracle(sh, data, O, L, rows=None, tol=1e-2, bf16_out=False):
    ref = orc.split_attention_fp8(sh, data["q"], data["k"], data["v"], rows=rows, tie_rel=TIE_REL)
    sel = slice(None) if rows is None else np.asarray(rows)
    for n in ("loc", "hist", "full"):
        got, r = O[n][:, sel], ref["O_" + n]
        for b in range(sh.B):
            for h in range(sh.H):
                rr = r[b, :, h]
                if np.all(rr == 0):
                    assert np.all(got[b, :, h] == 0), (n, b, h)
                    continue
                rms = np.sqrt(np.mean(rr ** 2))
                bound = tol * rms + ref["A_" + n][b, :, h] + (2.0 ** -8 * np.abs(rr) if bf16_out else 0.0)
                err = np.abs(got[b, :, h] - rr)
                assert np.all(err <= bound), (n, b, h, float((err / rms).max()))
        assert_lse(L[n][:, sel], ref["L_" + n], 1e-3)
    return ref


@pytest.mark.parametrize("idx", range(len(SHAPES)))
def test_fp8_attention_matches_the_fp8_oracle(idx):
    sh = SHAPES[idx]
    data = si.iid_qkv(sh, "bf16", ("gpu", "fp8", idx))
    O, L = run_fp8(sh, data)
    check_against_oracle(sh, data, O, L)
    # and the 8-bit attention stays close to the exact attention of the bf16 inputs
    exact = orc.split_attention(sh, data["q"], data["k"], data["v"])
    d = rel_fro(O["full"], exact["O_full"])
    print(f"fp8 vs exact (layout {idx}): relative Frobenius {d:.3e}")
    assert d <= 0.1, d


def test_fp8_attention_bf16_outputs_and_scaled_heads():
    """bf16 outputs; heads far from unit scale (Q x 2^10, K x 2^-12, V x 2^20 on
    different heads: the per-head scales absorb them)."""
    sh = SHAPES[0]
    data = si.iid_qkv(sh, "bf16", ("gpu", "fp8s"))
    data["q"] = si.round_to_bf16(data["q"] * np.array([1.0, 2.0 ** 10], np.float32)[None, None, :, None])
    data["k"] = si.round_to_bf16(data["k"] * np.array([2.0 ** -12, 1.0], np.float32)[None, None, :, None])
    data["v"] = si.round_to_bf16(data["v"] * np.array([2.0 ** 20, 1.0], np.float32)[None, None, :, None])
    O, L = run_fp8(sh, data, ispa.ISPA_BF16)
    check_against_oracle(sh, data, O, L, bf16_out=True)


def test_fp8_prepare_incremental_equals_fresh():
    """Frames prepared chunk by chunk -- the second chunk raising two heads' amax, so
    their rows are converted again with the new scale -- give the same outputs, bit
    for bit, as one prepare of the final K/V."""
    sh = SHAPES[0]
    data = si.iid_qkv(sh, "bf16", ("gpu", "fp8inc"))
    rows = slice(sh.cur_begin * sh.tpf, sh.cur_end * sh.tpf)
    k_new, v_new = data["k"].copy(), data["v"].copy()
    k_new[1, rows, 0] *= np.float32(8.0)
    v_new[0, rows, 1] *= np.float32(16.0)
    final = dict(data, k=si.round_to_bf16(k_new), v=si.round_to_bf16(v_new))

    def incremental(desc, k, v, kv8):
        ispa.ispa_kv8_prepare(desc, dev(data["k"], torch.bfloat16), dev(data["v"], torch.bfloat16), 0,
                              sh.kv_frames, kv8)
        ispa.ispa_kv8_prepare(desc, k, v, sh.cur_begin, sh.cur_end, kv8)

    O1, L1 = run_fp8(sh, final, prepare=incremental)
    O2, L2 = run_fp8(sh, final)
    for n in O1:
        assert np.array_equal(O1[n], O2[n]) and np.array_equal(L1[n], L2[n]), n
    check_against_oracle(sh, final, O1, L1)


def test_fp8_post_switch_full_size_1p3b_sampled_rows():
    """The post-switch attention in fp8 at the 1.3B size: the L-layer on its evicted
    K/V (sink + current, 9360 keys) and the F-layer over all 32760 keys, sampled rows
    against the fp8 oracle."""
    sh = si.SHAPE_1P3B
    data = si.iid_qkv(sh, "bf16", ("gpu", "fp8post"))
    rows = np.r_[0, 1, 1559, 1560, 3000, 4600:4680:20, 4679]
    # L-layer: the evicted layout's local group
    es = orc.evicted_shape(sh)
    ev = {"q": data["q"], "k": orc.evict_history(sh, data["k"]).astype(np.float32),
          "v": orc.evict_history(sh, data["v"]).astype(np.float32)}
    O, L = run_fp8(es, ev, ispa.ISPA_BF16)
    ref = orc.split_attention_fp8(es, ev["q"], ev["k"], ev["v"], rows=rows, tie_rel=TIE_REL)
    for b in range(sh.B):
        for h in range(sh.H):
            r = ref["O_loc"][b, :, h]
            err = np.abs(O["loc"][b, rows, h] - r)
            assert np.all(err <= 1e-2 * np.sqrt(np.mean(r ** 2)) + ref["A_loc"][b, :, h] + 2.0 ** -8 * np.abs(r)), (b, h)
    assert_lse(L["loc"][:, rows], ref["L_loc"], 1e-3)
    # F-layer: one group over every frame
    shF = dataclasses.replace(sh, sink_frames=sh.cur_begin, hist_begin=0, hist_end=0)
    O, L = run_fp8(shF, data, ispa.ISPA_BF16)
    ref = orc.split_attention_fp8(shF, data["q"], data["k"], data["v"], rows=rows, tie_rel=TIE_REL)
    for b in range(sh.B):
        for h in range(sh.H):
            r = ref["O_loc"][b, :, h]
            err = np.abs(O["loc"][b, rows, h] - r)
            assert np.all(err <= 1e-2 * np.sqrt(np.mean(r ** 2)) + ref["A_loc"][b, :, h] + 2.0 ** -8 * np.abs(r)), (b, h)
    assert_lse(L["loc"][:, rows], ref["L_loc"], 1e-3)


def test_fp8_local_projection_equals_attention_then_product():
    """ispa_attn_local_proj on a prepared fp8 K/V: the fp8 attention followed by the
    bf16 projection, bit for bit the two steps done separately."""
    sh = si.AttnShape(B=1, H=2, d=128, tpf=64, sink_frames=1, hist_begin=1, hist_end=4, cur_begin=4, cur_end=6,
                      kv_frames=6)
    data = si.iid_qkv(sh, "bf16", ("gpu", "fp8proj"))
    q, k, v = (dev(data[n], torch.bfloat16) for n in ("q", "k", "v"))
    D = sh.D
    W = dev(si.projection_weight(D, D, ("gpu", "fp8proj"), "bf16"), torch.bfloat16)
    desc = ispa.attn_desc(sh, ispa.ISPA_BF16, ispa.ISPA_BF16)
    pd = ispa.prepared(desc, ispa.ISPA_KV_E4M3_PREPARED)
    kv8 = torch.empty(ispa.ispa_kv8_bytes(desc), dtype=torch.uint8, device="cuda")
    ispa.ispa_kv8_prepare(desc, k, v, 0, sh.kv_frames, kv8)
    ws = torch.empty(ispa.ispa_attn_local_proj_workspace_bytes(pd), dtype=torch.uint8, device="cuda")
    y = nan_like((sh.B, sh.Lq, D), torch.float32)
    ispa.ispa_attn_local_proj(pd, q, kv8, None, W, D, y, ispa.ISPA_F32, ws)
    o = nan_like((sh.B, sh.Lq, sh.H, 128), torch.bfloat16)
    lse = nan_like((sh.B, sh.Lq, sh.H), torch.float32)
    ws2 = torch.empty(ispa.ispa_attn_split_workspace_bytes(pd), dtype=torch.uint8, device="cuda")
    ispa.ispa_attn_split(pd, q, kv8, None, o, lse, workspace=ws2)
    y2 = nan_like((sh.B * sh.Lq, D), torch.float32)
    ispa.ispa_gemm_bf16(sh.B * sh.Lq, D, D, o.reshape(sh.B * sh.Lq, D), W, y2, ispa.ISPA_F32)
    ispa.ispa_check_device_error()
    assert torch.equal(y.reshape(-1, D), y2)


def test_fp8_post_switch_full_size_14b_sampled_rows():
    """The F-layer in fp8 at the 14B size: 40 heads, all 102 960 keys of a drift
    history as one group, 1480 query tiles; sampled rows of two heads (the first
    and the last: the per-head scales make heads independent) against the fp8
    oracle of those heads."""
    sh = si.SHAPE_14B
    key = ("gpu", "fp8-14b")
    prefix = si.drift_layer_kv(sh, "bf16", 0, key)
    cq = si.chunk_qkv(sh, "bf16", 0, 0, key)
    data = {"q": cq["q"], "k": si.assemble_kv(prefix["k"], cq["k"], sh),
            "v": si.assemble_kv(prefix["v"], cq["v"], sh)}
    del prefix
    shF = dataclasses.replace(sh, sink_frames=sh.cur_begin, hist_begin=0, hist_end=0)
    O, L = run_fp8(shF, data, ispa.ISPA_BF16)
    heads = [0, sh.H - 1]
    sub = {n: np.ascontiguousarray(data[n][:, :, heads]) for n in ("q", "k", "v")}
    del data
    rows = np.r_[0, 1, 127, 128, 2339, 4608:4680:24, 4679]
    ref = orc.split_attention_fp8(dataclasses.replace(shF, H=len(heads)), sub["q"], sub["k"], sub["v"], rows=rows,
                                  tie_rel=TIE_REL)
    for b in range(sh.B):
        for x, h in enumerate(heads):
            r = ref["O_loc"][b, :, x]
            err = np.abs(O["loc"][b, rows, h] - r)
            assert np.all(err <= 1e-2 * np.sqrt(np.mean(r ** 2)) + ref["A_loc"][b, :, x] + 2.0 ** -8 * np.abs(r)), (b, h)
    assert_lse(L["loc"][:, rows][:, :, heads], ref["L_loc"], 1e-3)
