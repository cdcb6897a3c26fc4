"""Prepared fp16 V (ispa_v16_prepare): the attention on a kept, incrementally
updated copy equals the attention that converts V on every call, bit for bit,
and the oracle within the bf16 tolerances."""
import numpy as np
import pytest
import torch

import kv_cache_compression_two_b200 as ispa
import synth_inputs as si
from oracle import ispa_oracle as orc
from gpu_helpers import assert_lse, dev, host, max_over_rms, nan_like

pytestmark = pytest.mark.gpu

SHAPES = [
    si.AttnShape(B=2, H=3, d=128, tpf=40, sink_frames=1, hist_begin=1, hist_end=5, cur_begin=5, cur_end=7,
                 kv_frames=7),
    si.AttnShape(B=1, H=2, d=128, tpf=128, sink_frames=2, hist_begin=2, hist_end=8, cur_begin=8, cur_end=9,
                 kv_frames=9),
    si.AttnShape(B=1, H=1, d=128, tpf=200, sink_frames=2, hist_begin=2, hist_end=2, cur_begin=0, cur_end=2,
                 kv_frames=2),
]


def _split(desc, q, k, v, ws=None):
    sh_B, H = desc.B, desc.H
    Lq = (desc.cur_end - desc.cur_begin) * desc.tokens_per_frame
    o = {n: nan_like((sh_B, Lq, H, 128), torch.float32) for n in ("loc", "hist", "full")}
    l = {n: nan_like((sh_B, Lq, H), torch.float32) for n in ("loc", "hist", "full")}
    need = ispa.ispa_attn_split_workspace_bytes(desc)
    if need:
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    ispa.ispa_attn_split(desc, q, k, v, o["loc"], l["loc"], o["hist"], l["hist"], o["full"], l["full"], workspace=ws)
    ispa.ispa_check_device_error()
    return o, l


def _same(a, b):
    for n in a:
        assert torch.equal(a[n], b[n]) or (torch.isnan(a[n]).all() and torch.isnan(b[n]).all()), n


def _v_with_scaled_heads(sh, key):
    data = si.iid_qkv(sh, "bf16", key)
    v = data["v"].copy()
    if sh.H >= 2:
        v[0, :, 0] *= np.float32(2.0 ** 17)          # beyond the fp16 range: a negative exponent
        v[-1, :, 1] *= np.float32(2.0 ** -20)        # tiny: a positive exponent
    data["v"] = si.round_to_bf16(v)
    return data


@pytest.mark.parametrize("idx", range(len(SHAPES)))
def test_prepared_v_equals_per_call_conversion(idx):
    sh = SHAPES[idx]
    data = _v_with_scaled_heads(sh, ("gpu", "v16", idx))
    q, k, v = (dev(data[n], torch.bfloat16) for n in ("q", "k", "v"))
    desc = ispa.attn_desc(sh, ispa.ISPA_BF16, ispa.ISPA_F32)
    pdesc = ispa.prepared(desc)
    assert ispa.ispa_attn_split_workspace_bytes(pdesc) == 0
    v16 = torch.empty(ispa.ispa_v16_bytes(desc), dtype=torch.uint8, device="cuda")
    ispa.ispa_v16_prepare(desc, v, 0, sh.kv_frames, v16)
    o_ref, l_ref = _split(desc, q, k, v)
    o, l = _split(pdesc, q, k, v16)
    _same(o, o_ref)
    _same(l, l_ref)
    ref = orc.split_attention(sh, data["q"], data["k"], data["v"])
    for n in ("loc", "full"):
        got, r = host(o[n]), ref["O_" + n]
        for b in range(sh.B):
            for h in range(sh.H):
                rms = np.sqrt(np.mean(r[b, :, h] ** 2))
                assert np.abs(got[b, :, h] - r[b, :, h]).max() <= 1e-2 * rms, (n, b, h)
        assert_lse(host(l[n]), ref["L_" + n], 1e-3)


def test_prepared_v_incremental_chunks():
    """A growing cache: the whole buffer prepared once, then per chunk only the
    current frames are written and prepared.  The second chunk's new frames
    push one head past the fp16 range, so that head is converted again with a
    new exponent; both chunks equal the per-call conversion bit for bit."""
    sh = SHAPES[0]
    desc = ispa.attn_desc(sh, ispa.ISPA_BF16, ispa.ISPA_F32)
    pdesc = ispa.prepared(desc)
    data = si.iid_qkv(sh, "bf16", ("gpu", "v16inc"))
    q, k, v = (dev(data[n], torch.bfloat16) for n in ("q", "k", "v"))
    v16 = torch.empty(ispa.ispa_v16_bytes(desc), dtype=torch.uint8, device="cuda")
    ispa.ispa_v16_prepare(desc, v, 0, sh.kv_frames, v16)
    rows = slice(sh.cur_begin * sh.tpf, sh.cur_end * sh.tpf)
    for chunk in range(2):
        new = si.chunk_qkv(sh, "bf16", 0, chunk, ("gpu", "v16inc"))
        vn = new["v"].copy()
        if chunk == 1:
            vn[1, :, 2] *= np.float32(2.0 ** 16)
        vn = si.round_to_bf16(vn)
        v[:, rows] = dev(vn, torch.bfloat16)
        k[:, rows] = dev(new["k"], torch.bfloat16)
        q = dev(new["q"], torch.bfloat16)
        ispa.ispa_v16_prepare(desc, v, sh.cur_begin, sh.cur_end, v16)
        o, l = _split(pdesc, q, k, v16)
        o_ref, l_ref = _split(desc, q, k, v)
        _same(o, o_ref)
        _same(l, l_ref)
        full_v = host(v).astype(np.float32)
        ref = orc.split_attention(sh, host(q).astype(np.float32), host(k).astype(np.float32), full_v)
        got, r = host(o["full"]), ref["O_full"]
        for b in range(sh.B):
            for h in range(sh.H):
                rms = np.sqrt(np.mean(r[b, :, h] ** 2))
                assert np.abs(got[b, :, h] - r[b, :, h]).max() <= 1e-2 * rms, (chunk, b, h)


def test_prepared_v_eviction_and_post_switch():
    """An L-layer's prepared V is evicted with its state: local attention and the
    post-switch projection on it equal the calls on the evicted bf16 V."""
    sh = si.AttnShape(B=2, H=2, d=128, tpf=45, sink_frames=2, hist_begin=2, hist_end=6, cur_begin=6, cur_end=8,
                      kv_frames=9)
    data = _v_with_scaled_heads(sh, ("gpu", "v16ev"))
    desc = ispa.attn_desc(sh, ispa.ISPA_BF16, ispa.ISPA_BF16)
    pdesc = ispa.prepared(desc)
    k, v = dev(data["k"], torch.bfloat16), dev(data["v"], torch.bfloat16)
    v16 = torch.empty(ispa.ispa_v16_bytes(desc), dtype=torch.uint8, device="cuda")
    ispa.ispa_v16_prepare(desc, v, 0, sh.kv_frames, v16)
    ed, ped = ispa.ispa_kv_evicted_desc(desc), ispa.ispa_kv_evicted_desc(pdesc)
    assert ped.v_layout == ispa.ISPA_V_F16_PREPARED and ed.kv_frames == ped.kv_frames
    shape_ev = (sh.B, ed.kv_frames * sh.tpf, sh.H, sh.d)
    k_ev, v_ev = nan_like(shape_ev, torch.bfloat16), nan_like(shape_ev, torch.bfloat16)
    ispa.ispa_kv_evict_history(desc, k, v, k_ev, v_ev)
    k_ev2 = nan_like(shape_ev, torch.bfloat16)
    v16_ev = torch.empty(ispa.ispa_v16_bytes(ed), dtype=torch.uint8, device="cuda")
    ispa.ispa_kv_evict_history(pdesc, k, v16, k_ev2, v16_ev)
    assert torch.equal(k_ev, k_ev2)
    q = dev(data["q"], torch.bfloat16)
    D = sh.D
    W = dev(si.projection_weight(D, D, ("gpu", "v16ev"), "bf16"), torch.bfloat16)
    ys = []
    for d_, vv in ((ed, v_ev), (ped, v16_ev)):
        ws = torch.empty(ispa.ispa_attn_local_proj_workspace_bytes(d_), dtype=torch.uint8, device="cuda")
        y = nan_like((sh.B, sh.Lq, D), torch.float32)
        ispa.ispa_attn_local_proj(d_, q, k_ev, vv, W, D, y, ispa.ISPA_F32, ws)
        ispa.ispa_check_device_error()
        ys.append(y)
    assert torch.equal(ys[0], ys[1])
    # and the local attention itself against the oracle of the original layout
    o = nan_like((sh.B, sh.Lq, sh.H, sh.d), torch.float32)
    lse = nan_like((sh.B, sh.Lq, sh.H), torch.float32)
    ped32 = ispa.ispa_kv_evicted_desc(ispa.prepared(ispa.attn_desc(sh, ispa.ISPA_BF16, ispa.ISPA_F32)))
    ispa.ispa_attn_split(ped32, q, k_ev, v16_ev, o, lse, None, None, None, None)
    ispa.ispa_check_device_error()
    ref = orc.split_attention(sh, data["q"], data["k"], data["v"])
    got = host(o)
    for b in range(sh.B):
        for h in range(sh.H):
            r = ref["O_loc"][b, :, h]
            assert np.abs(got[b, :, h] - r).max() <= 1e-2 * np.sqrt(np.mean(r ** 2)), (b, h)
    assert_lse(host(lse), ref["L_loc"], 1e-3)


def test_prepared_v_fused_warmup_equals_plain():
    sh = SHAPES[0]
    data = si.iid_qkv(sh, "bf16", ("gpu", "v16fw"))
    q, k, v = (dev(data[n], torch.bfloat16) for n in ("q", "k", "v"))
    D = sh.D
    W = dev(si.projection_weight(D, D, ("gpu", "v16fw")))
    desc = ispa.attn_desc(sh, ispa.ISPA_BF16, ispa.ISPA_F32)
    pdesc = ispa.prepared(desc)
    v16 = torch.empty(ispa.ispa_v16_bytes(desc), dtype=torch.uint8, device="cuda")
    ispa.ispa_v16_prepare(desc, v, 0, sh.kv_frames, v16)
    out = []
    for d_, vv in ((desc, v), (pdesc, v16)):
        o = nan_like((sh.B, sh.Lq, sh.H, 128), torch.float32)
        l = nan_like((sh.B, sh.Lq, sh.H), torch.float32)
        G, C = torch.zeros((D, D), device="cuda"), torch.zeros((D, D), device="cuda")
        r2 = torch.zeros(1, dtype=torch.float64, device="cuda")
        ws = torch.empty(ispa.ispa_warmup_fused_workspace_bytes(d_, D), dtype=torch.uint8, device="cuda")
        ispa.ispa_warmup_fused(d_, q, k, vv, W, D, o, l, G, C, r2, ws)
        ispa.ispa_check_device_error()
        out.append((o, l, G, C, r2))
    assert ispa.ispa_warmup_fused_workspace_bytes(pdesc, D) < ispa.ispa_warmup_fused_workspace_bytes(desc, D)
    for a, b in zip(out[0][:4], out[1][:4]):
        assert torch.equal(a, b)
    assert abs(out[0][4].item() - out[1][4].item()) <= 1e-12 * abs(out[0][4].item())


def test_prepare_validation():
    sh = SHAPES[0]
    desc = ispa.attn_desc(sh, ispa.ISPA_BF16, ispa.ISPA_F32)
    v = torch.zeros((sh.B, sh.Lkv, sh.H, 128), dtype=torch.bfloat16, device="cuda")
    v16 = torch.empty(ispa.ispa_v16_bytes(desc), dtype=torch.uint8, device="cuda")
    with pytest.raises(ispa.IspaError):
        ispa.ispa_v16_prepare(desc, v, 3, 2, v16)                       # empty-reversed range
    with pytest.raises(ispa.IspaError):
        ispa.ispa_v16_prepare(desc, v, 0, sh.kv_frames + 1, v16)        # past the buffer
    f32 = ispa.attn_desc(sh, ispa.ISPA_F32, ispa.ISPA_F32)
    assert ispa.ispa_v16_bytes(f32) == 0
    with pytest.raises(ispa.IspaError):
        ispa.ispa_v16_prepare(f32, v, 0, 1, v16)
