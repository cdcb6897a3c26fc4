"""GPU parity of the two-group attention (and its fused merge) against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import kv_cache_compression_two_b200 as ispa
import synth_inputs as si
from oracle import ispa_oracle as orc
from gpu_helpers import assert_bf16_out, assert_lse, dev, host, max_over_rms, nan_like, normwise

pytestmark = pytest.mark.gpu


def run_split(shape, in_dt, out_dt, key, fused=True, want_hist=True):
    data = si.iid_qkv(shape, "bf16" if in_dt == ispa.ISPA_BF16 else "f32", key)
    tin = torch.bfloat16 if in_dt == ispa.ISPA_BF16 else torch.float32
    tout = torch.bfloat16 if out_dt == ispa.ISPA_BF16 else torch.float32
    q, k, v = dev(data["q"], tin), dev(data["k"], tin), dev(data["v"], tin)
    B, Lq, H, d = shape.B, shape.Lq, shape.H, shape.d
    o = {n: nan_like((B, Lq, H, d), tout) for n in ("loc", "hist", "full")}
    l = {n: nan_like((B, Lq, H), torch.float32) for n in ("loc", "hist", "full")}
    desc = ispa.attn_desc(shape, in_dt, out_dt)
    ws = torch.empty(max(1, ispa.ispa_attn_split_workspace_bytes(desc)), dtype=torch.uint8, device="cuda")
    ispa.ispa_attn_split(desc, q, k, v, o["loc"], l["loc"], o["hist"] if want_hist else None,
                         l["hist"] if want_hist else None, o["full"] if fused else None, l["full"] if fused else None,
                         workspace=ws)
    ispa.ispa_check_device_error()
    torch.cuda.synchronize()
    return data, {n: host(t) for n, t in o.items()}, {n: host(t) for n, t in l.items()}


def check(shape, data, O, L, in_dt, out_dt, fused=True, rows=None, want_hist=True):
    ref = orc.split_attention(shape, data["q"], data["k"], data["v"], rows=rows)
    names = ["loc"] + (["hist"] if want_hist else []) + (["full"] if fused else [])
    sel = slice(None) if rows is None else np.asarray(rows)
    for n in names:
        got_o, got_l = O[n][:, sel], L[n][:, sel]
        ref_o, ref_l = ref["O_" + n], ref["L_" + n]
        if in_dt == ispa.ISPA_F32:
            if np.abs(ref_o).max() > 0:
                assert normwise(got_o, ref_o) <= 1e-5, (n, normwise(got_o, ref_o))
            else:
                assert np.all(got_o == 0)
            assert_lse(got_l, ref_l, 1e-5 * max(1.0, float(np.abs(ref_l[np.isfinite(ref_l)]).max(initial=1.0))))
        else:
            if np.all(ref_o == 0):
                assert np.all(got_o == 0), n
            elif out_dt == ispa.ISPA_BF16:
                assert_bf16_out(got_o, ref_o)
            else:
                assert max_over_rms(got_o, ref_o) <= 1e-2, (n, max_over_rms(got_o, ref_o))
            assert_lse(got_l, ref_l, 1e-3)


# ---------------------------------------------------------------- fp32 (CUDA cores)
def test_tiny_fp32_matches_oracle():
    sh = si.TINY
    for chunk in range(4):
        data, O, L = run_split(sh, ispa.ISPA_F32, ispa.ISPA_F32, ("gpu", "tiny", chunk))
        check(sh, data, O, L, ispa.ISPA_F32, ispa.ISPA_F32)


@pytest.mark.parametrize("d", [32, 64, 128])
def test_fp32_random_layouts(d):
    g = np.random.default_rng(100 + d)
    for trial in range(4):
        sh = si.random_groups_shape(g, max_frames=6, d=d)
        data, O, L = run_split(sh, ispa.ISPA_F32, ispa.ISPA_F32, ("gpu", "f32rand", d, trial))
        check(sh, data, O, L, ispa.ISPA_F32, ispa.ISPA_F32)


# ---------------------------------------------------------------- bf16 (tcgen05)
BF16_SHAPES = [
    # several query tiles with a ragged tail, local group split in two ranges, ragged KV tiles
    si.AttnShape(B=2, H=2, d=128, tpf=50, sink_frames=2, hist_begin=2, hist_end=7, cur_begin=7, cur_end=10,
                 kv_frames=10),
    # no history: full == local, empty history group
    si.AttnShape(B=1, H=3, d=128, tpf=37, sink_frames=1, hist_begin=1, hist_end=1, cur_begin=1, cur_end=5,
                 kv_frames=5),
    # first chunk: the sink is the current chunk itself (one merged local range)
    si.AttnShape(B=1, H=1, d=128, tpf=200, sink_frames=2, hist_begin=2, hist_end=2, cur_begin=0, cur_end=2,
                 kv_frames=2),
    # exact multiples of the 128 tiles, long history
    si.AttnShape(B=1, H=2, d=128, tpf=128, sink_frames=1, hist_begin=1, hist_end=9, cur_begin=9, cur_end=10,
                 kv_frames=10),
    # single-token frames
    si.AttnShape(B=3, H=1, d=128, tpf=1, sink_frames=1, hist_begin=1, hist_end=40, cur_begin=40, cur_end=43,
                 kv_frames=43),
]


@pytest.mark.parametrize("idx", range(len(BF16_SHAPES)))
def test_bf16_layouts_fp32_out(idx):
    sh = BF16_SHAPES[idx]
    data, O, L = run_split(sh, ispa.ISPA_BF16, ispa.ISPA_F32, ("gpu", "bf16", idx))
    check(sh, data, O, L, ispa.ISPA_BF16, ispa.ISPA_F32)


@pytest.mark.parametrize("idx", [0, 1])
def test_bf16_layouts_bf16_out(idx):
    sh = BF16_SHAPES[idx]
    data, O, L = run_split(sh, ispa.ISPA_BF16, ispa.ISPA_BF16, ("gpu", "bf16o", idx))
    check(sh, data, O, L, ispa.ISPA_BF16, ispa.ISPA_BF16)


def test_bf16_optional_outputs():
    sh = BF16_SHAPES[0]
    data, O, L = run_split(sh, ispa.ISPA_BF16, ispa.ISPA_F32, ("gpu", "opt"), fused=False, want_hist=True)
    check(sh, data, O, L, ispa.ISPA_BF16, ispa.ISPA_F32, fused=False)
    assert np.all(np.isnan(O["full"]))  # untouched
    data, O, L = run_split(sh, ispa.ISPA_BF16, ispa.ISPA_F32, ("gpu", "opt2"), fused=True, want_hist=False)
    check(sh, data, O, L, ispa.ISPA_BF16, ispa.ISPA_F32, fused=True, want_hist=False)
    assert np.all(np.isnan(O["hist"]))


def test_bf16_v_outside_the_fp16_range():
    """Heads whose V the unscaled fp16 copy does not serve (|v| up to ~2^20; RMS ~2^-20) take
    the power-of-two-scaled copy; the others, one of them holding a few entries of 2^-19, stay
    unscaled.  Each (instance, head) is checked against the oracle relative to its own output
    scale."""
    sh = si.AttnShape(B=2, H=3, d=128, tpf=40, sink_frames=1, hist_begin=1, hist_end=5, cur_begin=5, cur_end=7,
                      kv_frames=7)
    data = si.iid_qkv(sh, "bf16", ("gpu", "vrange"))
    v = data["v"].copy()
    v[0, :, 0] *= np.float32(2.0 ** 17)     # largest |v| ~ 5 * 2^17 > 65504
    v[1, :, 2] *= np.float32(2.0 ** -20)    # nonzero |v| below 2^-17
    v[1, 5, 1] = np.float32(2.0 ** -19)     # one tiny entry in an otherwise normal head
    data["v"] = si.round_to_bf16(v)
    q, k, vv = dev(data["q"], torch.bfloat16), dev(data["k"], torch.bfloat16), dev(data["v"], torch.bfloat16)
    o = {n: nan_like((sh.B, sh.Lq, sh.H, 128), torch.float32) for n in ("loc", "hist", "full")}
    l = {n: nan_like((sh.B, sh.Lq, sh.H), torch.float32) for n in ("loc", "hist", "full")}
    desc = ispa.attn_desc(sh, ispa.ISPA_BF16, ispa.ISPA_F32)
    ws = torch.empty(ispa.ispa_attn_split_workspace_bytes(desc), dtype=torch.uint8, device="cuda")
    ispa.ispa_attn_split(desc, q, k, vv, o["loc"], l["loc"], o["hist"], l["hist"], o["full"], l["full"], workspace=ws)
    torch.cuda.synchronize()
    ref = orc.split_attention(sh, data["q"], data["k"], data["v"])
    for n in ("loc", "hist", "full"):
        got = host(o[n])
        for b in range(sh.B):
            for h in range(sh.H):
                r = ref["O_" + n][b, :, h]
                rms = np.sqrt(np.mean(r ** 2))
                assert np.abs(got[b, :, h] - r).max() <= 1e-2 * rms, (n, b, h)


def test_bf16_large_scores_and_rescaling():
    """Scores scaled up so the running maximum moves by far more than the rescale threshold."""
    sh = si.AttnShape(B=1, H=1, d=128, tpf=64, sink_frames=1, hist_begin=1, hist_end=6, cur_begin=6, cur_end=8,
                      kv_frames=8)
    data = si.iid_qkv(sh, "bf16", ("gpu", "big"))
    ramp = np.linspace(0.2, 3.0, sh.Lkv, dtype=np.float32)[None, :, None, None]
    data["k"] = si.round_to_bf16(data["k"] * ramp)
    q, k, v = dev(data["q"], torch.bfloat16), dev(data["k"], torch.bfloat16), dev(data["v"], torch.bfloat16)
    o = {n: nan_like((1, sh.Lq, 1, 128), torch.float32) for n in ("loc", "hist", "full")}
    l = {n: nan_like((1, sh.Lq, 1), torch.float32) for n in ("loc", "hist", "full")}
    desc = ispa.attn_desc(sh, ispa.ISPA_BF16, ispa.ISPA_F32)
    ws = torch.empty(ispa.ispa_attn_split_workspace_bytes(desc), dtype=torch.uint8, device="cuda")
    ispa.ispa_attn_split(desc, q, k, v, o["loc"], l["loc"], o["hist"], l["hist"], o["full"], l["full"], workspace=ws)
    torch.cuda.synchronize()
    check(sh, data, {n: host(t) for n, t in o.items()}, {n: host(t) for n, t in l.items()}, ispa.ISPA_BF16,
          ispa.ISPA_F32)


def test_bf16_fused_merge_equals_separate_merge():
    sh = BF16_SHAPES[0]
    data, O, L = run_split(sh, ispa.ISPA_BF16, ispa.ISPA_F32, ("gpu", "fm"))
    oa, ob = dev(O["loc"]), dev(O["hist"])
    la, lb = dev(L["loc"]), dev(L["hist"])
    oo, lo = torch.empty_like(oa), torch.empty_like(la)
    ispa.ispa_lse_merge(sh.B * sh.Lq, sh.H, 128, ispa.ISPA_F32, oa, la, ob, lb, oo, lo)
    torch.cuda.synchronize()
    assert np.abs(host(oo) - O["full"]).max() <= 1e-6 * np.abs(O["full"]).max()
    assert np.abs(host(lo) - L["full"]).max() <= 1e-5


def test_bf16_full_size_1p3b_sampled_rows():
    """The 1.3B-shaped layer (4680 queries, 32760 keys, 12 heads) at full size, sampled rows."""
    sh = si.SHAPE_1P3B
    data, O, L = run_split(sh, ispa.ISPA_BF16, ispa.ISPA_F32, ("gpu", "full1p3b"))
    rows = np.r_[0:3, 127:130, 2000:2003, 4600:4680:7, 4679]
    check(sh, data, O, L, ispa.ISPA_BF16, ispa.ISPA_F32, rows=rows)
    # unwritten outputs would still hold NaN
    for n in ("loc", "hist", "full"):
        assert not np.isnan(O[n]).any() and not np.isnan(L[n]).any()


# ---------------------------------------------------------------- KV eviction of post-switch L-layers
EVICT_LAYOUTS = [
    dict(sink_frames=2, hist_begin=2, hist_end=6, cur_begin=6, cur_end=8, kv_frames=9),  # sink | history | current | spare
    dict(sink_frames=0, hist_begin=0, hist_end=3, cur_begin=3, cur_end=5, kv_frames=5),  # no sink
    dict(sink_frames=5, hist_begin=0, hist_end=0, cur_begin=1, cur_end=3, kv_frames=6),  # current inside the sink
]


@pytest.mark.parametrize("layout", EVICT_LAYOUTS)
@pytest.mark.parametrize("in_dt", [ispa.ISPA_BF16, ispa.ISPA_F32])
def test_kv_evict_history_bit_exact(layout, in_dt):
    sh = si.AttnShape(B=2, H=3, d=128 if in_dt == ispa.ISPA_BF16 else 64, tpf=37, **layout)
    data = si.iid_qkv(sh, "bf16" if in_dt == ispa.ISPA_BF16 else "f32", ("gpu", "evict"))
    tin = torch.bfloat16 if in_dt == ispa.ISPA_BF16 else torch.float32
    k, v = dev(data["k"], tin), dev(data["v"], tin)
    desc = ispa.attn_desc(sh, in_dt, ispa.ISPA_F32)
    ed = ispa.ispa_kv_evicted_desc(desc)
    es = orc.evicted_shape(sh)
    assert (ed.kv_frames, ed.sink_frames, ed.cur_begin, ed.cur_end) == (es.kv_frames, es.sink_frames, es.cur_begin,
                                                                         es.cur_end)
    shape_out = (sh.B, ed.kv_frames * sh.tpf, sh.H, sh.d)
    k_out, v_out = nan_like(shape_out, tin), nan_like(shape_out, tin)
    ispa.ispa_kv_evict_history(desc, k, v, k_out, v_out)
    torch.cuda.synchronize()
    for got, name in ((k_out, "k"), (v_out, "v")):
        ref = orc.evict_history(sh, data[name])
        assert np.array_equal(host(got), ref.astype(np.float64)), name


@pytest.mark.parametrize("layout", EVICT_LAYOUTS[:2])
def test_attention_after_eviction_matches_oracle(layout):
    """The post-switch call on the evicted buffers attends to the same local
    entries: its local output and LSE match the oracle of the original layout."""
    sh = si.AttnShape(B=2, H=2, d=128, tpf=45, **layout)
    data = si.iid_qkv(sh, "bf16", ("gpu", "evict-attn"))
    desc = ispa.attn_desc(sh, ispa.ISPA_BF16, ispa.ISPA_F32)
    ed = ispa.ispa_kv_evicted_desc(desc)
    es = orc.evicted_shape(sh)
    k, v = dev(data["k"], torch.bfloat16), dev(data["v"], torch.bfloat16)
    shape_out = (sh.B, ed.kv_frames * sh.tpf, sh.H, sh.d)
    k_ev, v_ev = nan_like(shape_out, torch.bfloat16), nan_like(shape_out, torch.bfloat16)
    ispa.ispa_kv_evict_history(desc, k, v, k_ev, v_ev)
    del k, v
    q = dev(data["q"], torch.bfloat16)
    o = nan_like((sh.B, sh.Lq, sh.H, sh.d), torch.float32)
    lse = nan_like((sh.B, sh.Lq, sh.H), torch.float32)
    ws = torch.empty(max(1, ispa.ispa_attn_split_workspace_bytes(ed)), dtype=torch.uint8, device="cuda")
    ispa.ispa_attn_split(ed, q, k_ev, v_ev, o, lse, None, None, None, None, workspace=ws)
    ispa.ispa_check_device_error()
    torch.cuda.synchronize()
    ref = orc.split_attention(sh, data["q"], data["k"], data["v"])
    assert es.Lq == sh.Lq
    assert max_over_rms(host(o), ref["O_loc"]) <= 1e-2
    assert_lse(host(lse), ref["L_loc"], 1e-3)


def test_kv_eviction_releases_the_history_bytes():
    """Real eviction: once the caller frees the original K/V, the device
    allocator holds exactly the kept frames (sizes chosen as multiples of the
    allocator's 512-byte granule)."""
    layout = EVICT_LAYOUTS[0]
    sh = si.AttnShape(B=2, H=4, d=128, tpf=64, **layout)
    desc = ispa.attn_desc(sh, ispa.ISPA_BF16, ispa.ISPA_BF16)
    ed = ispa.ispa_kv_evicted_desc(desc)
    torch.cuda.synchronize()
    base = torch.cuda.memory_allocated()
    full = (sh.B, sh.kv_frames * sh.tpf, sh.H, sh.d)
    k = torch.ones(full, dtype=torch.bfloat16, device="cuda")
    v = torch.ones(full, dtype=torch.bfloat16, device="cuda")
    before = torch.cuda.memory_allocated() - base
    kept = (sh.B, ed.kv_frames * sh.tpf, sh.H, sh.d)
    k_ev = torch.empty(kept, dtype=torch.bfloat16, device="cuda")
    v_ev = torch.empty(kept, dtype=torch.bfloat16, device="cuda")
    ispa.ispa_kv_evict_history(desc, k, v, k_ev, v_ev)
    torch.cuda.synchronize()
    del k, v
    after = torch.cuda.memory_allocated() - base
    row_bytes = sh.H * sh.d * 2
    freed_per_tensor = sh.B * (sh.kv_frames - ed.kv_frames) * sh.tpf * row_bytes
    assert before == 2 * sh.B * sh.kv_frames * sh.tpf * row_bytes
    assert before - after == 2 * freed_per_tensor
    assert torch.all(k_ev == 1) and torch.all(v_ev == 1)


def test_post_switch_full_size_1p3b_sampled_rows():
    """The post-switch calls as the bench times them, on the 1.3B-shaped layer at full size: the
    L-layer on its evicted K/V (sink + current, 9360 keys) projected with W + dW, the F-layer over
    all 32760 keys projected with W; bf16 output, sampled rows against the oracle (the output
    tolerance of the bf16 projection, 2e-2 of RMS plus the bf16 output rounding)."""
    import dataclasses
    sh = si.SHAPE_1P3B
    D = sh.D
    data = si.iid_qkv(sh, "bf16", ("gpu", "post1p3b"))
    W = si.projection_weight(D, D, ("gpu", "post1p3b"), "bf16")
    dW = (1e-3 * si.rng("gpu", "post1p3b", "dW").standard_normal((D, D))).astype(np.float32)
    q = dev(data["q"], torch.bfloat16)
    k_full, v_full = dev(data["k"], torch.bfloat16), dev(data["v"], torch.bfloat16)
    rows = np.r_[0:2, 1559:1562, 3000, 4600:4680:9, 4679]
    for layer in ("L", "F"):
        if layer == "L":
            desc_full = ispa.attn_desc(sh, ispa.ISPA_BF16, ispa.ISPA_BF16)
            desc = ispa.ispa_kv_evicted_desc(desc_full)
            shape_ev = (sh.B, desc.kv_frames * sh.tpf, sh.H, sh.d)
            k, v = nan_like(shape_ev, torch.bfloat16), nan_like(shape_ev, torch.bfloat16)
            ispa.ispa_kv_evict_history(desc_full, k_full, v_full, k, v)
            Wp = si.round_to_bf16(W + dW)   # the absorbed weight as the layer holds it
            ref_sh = sh                     # local attention of the original layout
        else:
            ref_sh = dataclasses.replace(sh, sink_frames=sh.cur_begin, hist_begin=0, hist_end=0)
            desc = ispa.attn_desc(ref_sh, ispa.ISPA_BF16, ispa.ISPA_BF16)
            k, v, Wp = k_full, v_full, W
        ws = torch.empty(ispa.ispa_attn_local_proj_workspace_bytes(desc), dtype=torch.uint8, device="cuda")
        y = nan_like((sh.B, sh.Lq, D), torch.bfloat16)
        ispa.ispa_attn_local_proj(desc, q, k, v, dev(Wp, torch.bfloat16), D, y, ispa.ISPA_BF16, ws)
        ispa.ispa_check_device_error()
        torch.cuda.synchronize()
        got = host(y)
        assert not np.isnan(got).any(), layer
        ref = orc.local_projection(ref_sh, data["q"], data["k"], data["v"], Wp, None, rows=rows)
        assert_bf16_out(got[:, rows], ref, tol=2e-2)


@pytest.mark.parametrize("B,hist", [(2, 15), (1, 117)])
def test_bf16_sweep_extremes_sampled_rows(B, hist):
    """Points of the history / batch sweep at full size: the 1.3B layout with two
    instances, and with the longest history (117 frames, 191 880 keys), on the
    prepared V as the bench runs them; sampled rows of every instance against the
    oracle."""
    sh = si.video_shape(12, hist, B=B)
    data = si.iid_qkv(sh, "bf16", ("gpu", "sweep", B, hist))
    q, k, v = dev(data["q"], torch.bfloat16), dev(data["k"], torch.bfloat16), dev(data["v"], torch.bfloat16)
    desc = ispa.attn_desc(sh, ispa.ISPA_BF16, ispa.ISPA_F32)
    v16 = torch.empty(ispa.ispa_v16_bytes(desc), dtype=torch.uint8, device="cuda")
    ispa.ispa_v16_prepare(desc, v, 0, sh.kv_frames, v16)
    o = {n: nan_like((B, sh.Lq, sh.H, 128), torch.float32) for n in ("loc", "hist", "full")}
    l = {n: nan_like((B, sh.Lq, sh.H), torch.float32) for n in ("loc", "hist", "full")}
    ispa.ispa_attn_split(ispa.prepared(desc), q, k, v16, o["loc"], l["loc"], o["hist"], l["hist"], o["full"],
                         l["full"])
    ispa.ispa_check_device_error()
    torch.cuda.synchronize()
    rows = np.r_[0, 127, 1560, 3119, 4600:4680:16, 4679]
    check(sh, data, {n: host(t) for n, t in o.items()}, {n: host(t) for n, t in l.items()}, ispa.ISPA_BF16,
          ispa.ISPA_F32, rows=rows)
