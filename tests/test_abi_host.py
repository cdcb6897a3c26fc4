"""Host-side checks of the C ABI: the library loads, exports every entry point
declared in include/ispa.h, and rejects invalid arguments before touching the
GPU (no CUDA call is made on these paths, so they run without a GPU)."""
import ctypes
import os
import re

import pytest

import kv_cache_compression_two_b200 as ispa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    text = open(os.path.join(ROOT, "include", "ispa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ispa_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    L = ispa.lib()
    declared = header_functions()
    assert len(declared) >= 12
    for name in declared:
        assert hasattr(L, name), name
    assert set(declared) == set(ispa.EXPORTED)


def test_version_string():
    assert "sm_100a" in ispa.version()


def _desc(**kw):
    base = dict(B=1, H=2, head_dim=128, tokens_per_frame=16, sink_frames=1, hist_begin=1, hist_end=4, cur_begin=4,
                cur_end=5, kv_frames=5, in_dtype=ispa.ISPA_BF16, out_dtype=ispa.ISPA_F32, softmax_scale=0.0)
    base.update(kw)
    return ispa.AttnDesc(**base)


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first


def _split(desc, ptrs=None):
    p = ptrs or [FAKE] * 9
    return ispa.lib().ispa_attn_split(ctypes.byref(desc), *p, FAKE, 1 << 40, None)


@pytest.mark.parametrize("kw,frag", [
    (dict(head_dim=96), "head_dim"),
    (dict(B=0), "B, H"),
    (dict(kv_frames=0), "kv_frames"),
    (dict(cur_begin=5, cur_end=5), "current chunk"),
    (dict(cur_end=6), "current chunk"),
    (dict(hist_begin=0, hist_end=2), "overlaps"),
    (dict(hist_begin=3, hist_end=5), "overlaps"),
    (dict(sink_frames=6), "sink_frames"),
    (dict(in_dtype=7), "dtype"),
])
def test_attn_split_rejects_bad_layouts(kw, frag):
    st = _split(_desc(**kw))
    assert st == ispa.ISPA_ERR_INVALID_ARG
    assert frag in ispa.lib().ispa_last_error().decode()


def test_attn_split_rejects_null_and_misaligned():
    assert ispa.lib().ispa_attn_split(None, *([FAKE] * 9), FAKE, 1 << 40, None) == ispa.ISPA_ERR_INVALID_ARG
    # workspace too small for the bf16 path
    assert ispa.lib().ispa_attn_split(ctypes.byref(_desc()), *([FAKE] * 9), FAKE, 16, None) == ispa.ISPA_ERR_INVALID_ARG
    assert "workspace" in ispa.lib().ispa_last_error().decode()
    p = [FAKE] * 9
    p[0] = FAKE + 4
    assert _split(_desc(), p) == ispa.ISPA_ERR_INVALID_ARG
    p = [FAKE] * 9
    p[5] = None  # o_hist without lse_hist
    p[6] = FAKE
    p[5], p[6] = None, FAKE
    assert _split(_desc(), p) == ispa.ISPA_ERR_INVALID_ARG


def test_bf16_other_head_dims_unsupported():
    st = _split(_desc(head_dim=64))
    assert st == ispa.ISPA_ERR_UNSUPPORTED


def test_stats_and_ridge_validation():
    L = ispa.lib()
    assert L.ispa_accum_stats(10, 48, 64, *([FAKE] * 5), FAKE, ispa.ISPA_PREC_TF32, FAKE, 1 << 30,
                              None) == ispa.ISPA_ERR_INVALID_ARG  # D % 32
    assert L.ispa_accum_stats(10, 64, 64, *([FAKE] * 5), FAKE, ispa.ISPA_PREC_TF32, FAKE, 16,
                              None) == ispa.ISPA_ERR_INVALID_ARG  # workspace too small
    assert "workspace" in L.ispa_last_error().decode()
    assert L.ispa_ridge_solve(64, 64, FAKE, FAKE, FAKE, ctypes.c_float(-1.0), 0, 0, FAKE, FAKE, FAKE, 1 << 30,
                              None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_ridge_solve(64, 64, FAKE, FAKE, FAKE, ctypes.c_float(1.0), 0, 99, FAKE, FAKE, FAKE, 1 << 30,
                              None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_select_layers(4, FAKE, 5, FAKE, FAKE, None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_select_layers(5000, FAKE, 5, FAKE, FAKE, None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_lse_merge(10, 2, 12, ispa.ISPA_F32, *([FAKE] * 6), None) == ispa.ISPA_ERR_INVALID_ARG
    # lse_out overlapping lse_a is rejected (in-place O is allowed, in-place LSE is not)
    assert L.ispa_lse_merge(10, 2, 64, ispa.ISPA_F32, FAKE, FAKE, FAKE, FAKE + 4096, FAKE + 8192, FAKE,
                            None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_absorb_weight(3, 3, FAKE, 0, FAKE, FAKE, 0, None) == ispa.ISPA_ERR_INVALID_ARG


def test_workspace_queries():
    L = ispa.lib()
    D, Dout, T = 1536, 1536, 4680
    ridge = L.ispa_ridge_workspace_bytes(D, Dout)
    assert ridge >= 2 * D * Dout * 4
    tf32 = L.ispa_accum_stats_workspace_bytes(T, D, Dout, ispa.ISPA_PREC_TF32)
    assert tf32 >= (2 * T * D + D * Dout + T * Dout) * 4
    assert L.ispa_accum_stats_workspace_bytes(T, D, Dout, ispa.ISPA_PREC_F32) >= T * Dout * 4
    d = _desc(H=12, tokens_per_frame=1560, sink_frames=3, hist_begin=3, hist_end=18, cur_begin=18, cur_end=21,
              kv_frames=21)
    assert L.ispa_attn_local_proj_workspace_bytes(ctypes.byref(d)) >= 4680 * 1536 * 2 + 32760 * 1536 * 2
    assert L.ispa_attn_split_workspace_bytes(ctypes.byref(d)) >= 32760 * 1536 * 2
    d.in_dtype = ispa.ISPA_F32
    assert L.ispa_attn_split_workspace_bytes(ctypes.byref(d)) == 0
    assert L.ispa_ridge_workspace_bytes(0, 5) == 0


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    import importlib
    import sys
    monkeypatch.setattr(ispa, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(ispa, "_lib", None)
    with pytest.raises(ImportError):
        ispa.lib()


# ---------------------------------------------------------------- KV eviction (host side)
@pytest.mark.parametrize("layout", [
    dict(sink_frames=1, hist_begin=1, hist_end=4, cur_begin=4, cur_end=5, kv_frames=5),   # sink | history | current
    dict(sink_frames=2, hist_begin=2, hist_end=5, cur_begin=5, cur_end=8, kv_frames=10),  # frames after the chunk
    dict(sink_frames=0, hist_begin=0, hist_end=3, cur_begin=3, cur_end=5, kv_frames=5),   # no sink
    dict(sink_frames=3, hist_begin=0, hist_end=0, cur_begin=2, cur_end=4, kv_frames=4),   # current overlaps the sink
    dict(sink_frames=4, hist_begin=0, hist_end=0, cur_begin=4, cur_end=6, kv_frames=6),   # current right after the sink
    dict(sink_frames=5, hist_begin=0, hist_end=0, cur_begin=1, cur_end=3, kv_frames=6),   # current inside the sink
])
def test_kv_evicted_desc_matches_oracle_layout(layout):
    import synth_inputs as si
    from oracle import ispa_oracle as orc
    d = _desc(**layout)
    e = ispa.ispa_kv_evicted_desc(d)
    sh = si.AttnShape(B=d.B, H=d.H, d=d.head_dim, tpf=d.tokens_per_frame, **layout)
    es = orc.evicted_shape(sh)
    got = (e.sink_frames, e.hist_begin, e.hist_end, e.cur_begin, e.cur_end, e.kv_frames)
    assert got == (es.sink_frames, es.hist_begin, es.hist_end, es.cur_begin, es.cur_end, es.kv_frames)
    assert (e.B, e.H, e.head_dim, e.tokens_per_frame, e.in_dtype) == (d.B, d.H, d.head_dim, d.tokens_per_frame,
                                                                       d.in_dtype)


def test_kv_eviction_validation():
    L = ispa.lib()
    bad = _desc(cur_begin=5, cur_end=5)
    out = ispa.AttnDesc()
    assert L.ispa_kv_evicted_desc(ctypes.byref(bad), ctypes.byref(out)) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_kv_evicted_desc(ctypes.byref(_desc()), None) == ispa.ISPA_ERR_INVALID_ARG
    d = _desc()
    assert L.ispa_kv_evict_history(ctypes.byref(d), FAKE, FAKE, None, FAKE, None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_kv_evict_history(ctypes.byref(d), FAKE, FAKE, FAKE + 8, FAKE, None) == ispa.ISPA_ERR_INVALID_ARG
    # outputs overlapping the inputs are rejected (here k_out == k)
    assert L.ispa_kv_evict_history(ctypes.byref(d), FAKE, FAKE + (1 << 24), FAKE, FAKE + (1 << 26),
                                   None) == ispa.ISPA_ERR_INVALID_ARG
    assert "overlap" in L.ispa_last_error().decode()


def test_recalibration_validation():
    L = ispa.lib()
    assert L.ispa_stats_reset(0, 4, FAKE, FAKE, FAKE, None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_stats_reset(4, 4, None, FAKE, FAKE, None) == ispa.ISPA_ERR_INVALID_ARG
    d = _desc()
    assert L.ispa_kv_restore(ctypes.byref(d), FAKE, None, FAKE, FAKE, None) == ispa.ISPA_ERR_INVALID_ARG
    bad = _desc(cur_begin=5, cur_end=5)
    assert L.ispa_kv_restore(ctypes.byref(bad), FAKE, FAKE, FAKE + (1 << 24), FAKE + (1 << 26),
                             None) == ispa.ISPA_ERR_INVALID_ARG


def test_selftest_validation():
    L = ispa.lib()
    assert L.ispa_selftest_wait_timeout(10, None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_selftest_wait_timeout(20_000_000_000, None) == ispa.ISPA_ERR_INVALID_ARG


def test_w8a8_validation():
    L = ispa.lib()
    E8, I8, BAD = ispa.ISPA_Q8_E4M3, ispa.ISPA_Q8_INT8, 7
    inv = ispa.ISPA_ERR_INVALID_ARG
    a, b, c = FAKE, FAKE + (1 << 24), FAKE + (1 << 26)
    # K must be a positive multiple of 16; the format must be known
    assert L.ispa_quantize_rows(4, 24, a, E8, b, c, None) == inv
    assert L.ispa_quantize_rows(4, 0, a, E8, b, c, None) == inv
    assert L.ispa_quantize_rows(4, 32, a, BAD, b, c, None) == inv
    assert L.ispa_quantize_rows(-1, 32, a, I8, b, c, None) == inv
    assert L.ispa_quantize_rows(0, 32, None, I8, None, None, None) == ispa.ISPA_OK   # nothing to do
    assert L.ispa_quantize_rows(4, 32, a + 8, I8, b, c, None) == inv               # unaligned
    assert L.ispa_quantize_rows(4, 32, a, I8, a + 64, c, None) == inv              # q overlaps x
    assert L.ispa_quantize_weight(40, 8, a, E8, b, c, None) == inv
    assert L.ispa_quantize_weight(32, 8, a, E8, b, a + 16, None) == inv           # sw overlaps W
    assert L.ispa_quantize_weight(32, 8, None, E8, b, c, None) == inv
    # the product: N a multiple of 16, y apart from the inputs
    assert L.ispa_gemm_q8(4, 24, 32, a, b, c, c + 4096, E8, c + 8192, ispa.ISPA_BF16, None) == inv
    assert L.ispa_gemm_q8(4, 32, 40, a, b, c, c + 4096, E8, c + 8192, ispa.ISPA_BF16, None) == inv
    assert L.ispa_gemm_q8(4, 32, 32, a, b, c, c + 4096, BAD, c + 8192, ispa.ISPA_BF16, None) == inv
    assert L.ispa_gemm_q8(4, 32, 32, a, b, c, c + 4096, I8, c + 8192, 9, None) == inv
    assert L.ispa_gemm_q8(4, 32, 32, a, b, c, c + 4096, I8, a, ispa.ISPA_F32, None) == inv
    assert L.ispa_gemm_q8(0, 32, 32, None, None, None, None, I8, None, ispa.ISPA_F32, None) == ispa.ISPA_OK
    assert L.ispa_gemm_q8(4, 32, 131088, a, b, c, c + 4096, I8, c + 8192, ispa.ISPA_F32, None) == inv  # int32 range
    assert L.ispa_gemm_bf16(4, 24, 32, a, b, c, ispa.ISPA_BF16, None) == inv
    assert L.ispa_gemm_bf16(4, 32, 24, a, b, c, ispa.ISPA_BF16, None) == inv
    assert L.ispa_gemm_bf16(4, 32, 32, a, b, a + 32, ispa.ISPA_BF16, None) == inv   # y overlaps A
    assert L.ispa_gemm_bf16(0, 32, 32, None, None, None, ispa.ISPA_BF16, None) == ispa.ISPA_OK
    # the post-switch step: workspace covers the bf16 path plus the 8-bit rows and their scales
    d = _desc()
    base = L.ispa_attn_local_proj_workspace_bytes(ctypes.byref(d))
    need = L.ispa_attn_local_proj_q8_workspace_bytes(ctypes.byref(d))
    rows = d.B * (d.cur_end - d.cur_begin) * d.tokens_per_frame
    assert need >= base + rows * d.H * d.head_dim + rows * 4
    assert L.ispa_attn_local_proj_q8(ctypes.byref(d), a, a, a, b, c, E8, 48, c + 4096, ispa.ISPA_BF16, FAKE,
                                     need - 1, None) == inv
    assert L.ispa_attn_local_proj_q8(ctypes.byref(d), a, a, a, b, c, BAD, 48, c + 4096, ispa.ISPA_BF16, FAKE,
                                     need, None) == inv
    assert L.ispa_attn_local_proj_q8(ctypes.byref(d), a, a, a, b, c, I8, 40, c + 4096, ispa.ISPA_BF16, FAKE,
                                     need, None) == inv


def test_warmup_fused_validation():
    L = ispa.lib()
    inv = ispa.ISPA_ERR_INVALID_ARG
    d = _desc()
    need = L.ispa_warmup_fused_workspace_bytes(ctypes.byref(d), 64)
    T, D = d.B * (d.cur_end - d.cur_begin) * d.tokens_per_frame, d.H * d.head_dim
    assert need >= 2 * T * D * 4 + D * 64 * 4 + T * 64 * 4          # dA, Ar, W in tf32, R
    assert L.ispa_warmup_fused_workspace_bytes(ctypes.byref(d), 0) == 0
    args = [FAKE] * 3 + [FAKE, 64] + [FAKE] * 5
    assert L.ispa_warmup_fused(ctypes.byref(d), *args, FAKE, need - 1, None) == inv      # workspace short
    bad = list(args); bad[4] = 48                                                        # Dout % 32
    assert L.ispa_warmup_fused(ctypes.byref(d), *bad, FAKE, need, None) == inv
    bad = list(args); bad[9] = None                                                      # r2
    assert L.ispa_warmup_fused(ctypes.byref(d), *bad, FAKE, need, None) == inv
    d32 = _desc(in_dtype=ispa.ISPA_F32)
    assert L.ispa_warmup_fused(ctypes.byref(d32), *args, FAKE, need, None) == ispa.ISPA_ERR_UNSUPPORTED


def test_header_is_plain_c_and_links(tmp_path):
    """include/ispa.h compiles as C99 and a C program links against libispa.so and calls it:
    the boundary needs neither C++ nor torch (no GPU call: version, a rejected argument and the
    last-error text)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "probe.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "ispa.h"
int main(void) {
  const char *v = ispa_version();
  if (!v || !*v) return 2;
  ispa_status st = ispa_stats_reset(0, 4, NULL, NULL, NULL, NULL);
  if (st != ISPA_ERR_INVALID_ARG) return 3;
  if (strlen(ispa_last_error()) == 0) return 4;
  printf("%s\n", v);
  return 0;
}
''')
    lib_dir = os.path.join(ROOT, "kv_cache_compression_two_b200")
    exe = tmp_path / "probe"
    subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o",
                    str(exe), "-L", lib_dir, "-lispa", "-Wl,-rpath," + lib_dir], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, (out.returncode, out.stderr)
    assert out.stdout.strip() == ispa.lib().ispa_version().decode()


def test_descriptor_layout_matches_the_binding(tmp_path):
    """sizeof(ispa_attn_desc) and the offset of every field agree between the C header and the
    ctypes structure the binding passes."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    fields = [f for f, _ in ispa.AttnDesc._fields_]
    src = tmp_path / "layout.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "ispa.h"\nint main(void) {\n'
                   '  printf("%zu\\n", sizeof(ispa_attn_desc));\n' +
                   "".join(f'  printf("%zu\\n", offsetof(ispa_attn_desc, {f}));\n' for f in fields) +
                   "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    vals = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    assert vals[0] == ctypes.sizeof(ispa.AttnDesc)
    assert vals[1:] == [getattr(ispa.AttnDesc, f).offset for f in fields]


def test_prepare_and_error_entry_points_validate_on_the_host():
    L = ispa.lib()
    d = _desc()
    # prepared fp16 V / fp8 K/V: frame ranges and dtypes are checked before any launch
    assert L.ispa_v16_prepare(ctypes.byref(d), FAKE, 3, 2, FAKE, None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_v16_prepare(ctypes.byref(d), FAKE, 0, 6, FAKE, None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_kv8_prepare(ctypes.byref(d), FAKE, FAKE, 0, 9, FAKE, None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_kv8_prepare(ctypes.byref(d), FAKE, FAKE, 0, 1, FAKE, None) == ispa.ISPA_ERR_INVALID_ARG  # overlap
    f32 = _desc(in_dtype=ispa.ISPA_F32, head_dim=64)
    assert L.ispa_v16_bytes(ctypes.byref(f32)) == 0 and L.ispa_kv8_bytes(ctypes.byref(f32)) == 0
    assert L.ispa_v16_prepare(ctypes.byref(f32), FAKE, 0, 1, FAKE * 2, None) == ispa.ISPA_ERR_UNSUPPORTED
    assert L.ispa_v16_bytes(ctypes.byref(d)) > 5 * 16 * 2 * 128 * 2
    # a prepared layout needs bf16 inputs with head_dim 128; an unknown layout is rejected
    bad = _desc(in_dtype=ispa.ISPA_F32, head_dim=64, v_layout=ispa.ISPA_V_F16_PREPARED)
    assert _split(bad) == ispa.ISPA_ERR_INVALID_ARG
    assert _split(_desc(v_layout=7)) == ispa.ISPA_ERR_INVALID_ARG
    # the fp8 layout is not evicted (the bf16 K/V is), nor run by the fused warmup
    d8 = _desc(v_layout=ispa.ISPA_KV_E4M3_PREPARED)
    assert L.ispa_kv_evict_history(ctypes.byref(d8), FAKE, FAKE, FAKE * 2, FAKE * 3, None) == \
        ispa.ISPA_ERR_INVALID_ARG
    assert "evict" in L.ispa_last_error().decode()
    assert L.ispa_warmup_fused(ctypes.byref(d8), FAKE, FAKE, FAKE, FAKE, 256, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                               1 << 40, None) == ispa.ISPA_ERR_UNSUPPORTED
    # the epsilon entry point
    assert L.ispa_absorb_error(0, 4, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_absorb_error(64, 64, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16, None) == ispa.ISPA_ERR_INVALID_ARG
    assert L.ispa_absorb_error_workspace_bytes(64, 64) >= 64 * 64 * 4
