"""Python binding of libispa, the B200 (sm_100a) ISPA hot path.

Argument marshalling only: every step of the path runs in the CUDA kernels of
``libispa.so`` (built in-tree by :mod:`kv_cache_compression_two_b200.build`).
The first call into the library raises ImportError when it has not been
built; there is no CPU or PyTorch fallback.

Tensor arguments may be ``torch.Tensor`` objects (their ``data_ptr()`` is
passed; the binding checks device, dtype and contiguity) or raw integer device
addresses.  ``stream`` may be a ``torch.cuda.Stream``, a raw ``cudaStream_t``
integer or ``None`` (the current torch stream when torch is initialised,
otherwise the legacy default stream).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libispa.so")

ISPA_OK, ISPA_ERR_INVALID_ARG, ISPA_ERR_UNSUPPORTED, ISPA_ERR_CUDA, ISPA_ERR_NOT_SPD, ISPA_ERR_TIMEOUT = range(6)
ISPA_F32, ISPA_BF16 = 0, 1
ISPA_PREC_TF32, ISPA_PREC_F32 = 0, 1
ISPA_Q8_E4M3, ISPA_Q8_INT8 = 0, 1
ISPA_V_PLAIN, ISPA_V_F16_PREPARED, ISPA_KV_E4M3_PREPARED = 0, 1, 2

STATUS_NAMES = {0: "ISPA_OK", 1: "ISPA_ERR_INVALID_ARG", 2: "ISPA_ERR_UNSUPPORTED", 3: "ISPA_ERR_CUDA",
                4: "ISPA_ERR_NOT_SPD", 5: "ISPA_ERR_TIMEOUT"}

# Every entry point declared in include/ispa.h.
EXPORTED = ("ispa_version", "ispa_last_error", "ispa_launch_count", "ispa_check_device_error", "ispa_attn_split_workspace_bytes", "ispa_attn_split", "ispa_lse_merge",
            "ispa_accum_stats_workspace_bytes", "ispa_accum_stats", "ispa_ridge_workspace_bytes", "ispa_ridge_solve",
            "ispa_select_layers", "ispa_absorb_weight", "ispa_attn_local_proj_workspace_bytes",
            "ispa_attn_local_proj", "ispa_ridge_solve_noalloc", "ispa_kv_evicted_desc", "ispa_kv_evict_history",
            "ispa_kv_restore", "ispa_stats_reset", "ispa_selftest_wait_timeout", "ispa_quantize_rows",
            "ispa_quantize_weight", "ispa_gemm_q8", "ispa_gemm_bf16", "ispa_attn_local_proj_q8_workspace_bytes",
            "ispa_attn_local_proj_q8", "ispa_warmup_fused_workspace_bytes", "ispa_warmup_fused",
            "ispa_v16_bytes", "ispa_v16_prepare", "ispa_absorb_error_workspace_bytes", "ispa_absorb_error",
            "ispa_kv8_bytes", "ispa_kv8_prepare")
RIDGE_NOALLOC_MAX_D = RIDGE_NOALLOC_MAX_DOUT = 1024


class IspaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class AttnDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("tokens_per_frame", ctypes.c_int), ("sink_frames", ctypes.c_int), ("hist_begin", ctypes.c_int),
                ("hist_end", ctypes.c_int), ("cur_begin", ctypes.c_int), ("cur_end", ctypes.c_int),
                ("kv_frames", ctypes.c_int), ("in_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int),
                ("softmax_scale", ctypes.c_float), ("v_layout", ctypes.c_int)]


def attn_desc(shape, in_dtype: int, out_dtype: int, softmax_scale: float = 0.0,
              v_layout: int = ISPA_V_PLAIN) -> AttnDesc:
    """Builds an AttnDesc from any object with the frame-layout attributes (B, H, d, tpf, ...)."""
    return AttnDesc(shape.B, shape.H, shape.d, shape.tpf, shape.sink_frames, shape.hist_begin, shape.hist_end,
                    shape.cur_begin, shape.cur_end, shape.kv_frames, in_dtype, out_dtype, softmax_scale, v_layout)


def prepared(desc: AttnDesc, layout: int = ISPA_V_F16_PREPARED) -> AttnDesc:
    """A copy of desc whose V (ISPA_V_F16_PREPARED, ispa_v16_prepare) or K/V
    (ISPA_KV_E4M3_PREPARED, ispa_kv8_prepare) comes prepared."""
    d = AttnDesc.from_buffer_copy(desc)
    d.v_layout = layout
    return d


_lib = None
_vp, _ci, _cf, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t


def lib() -> ctypes.CDLL:
    """Loads libispa.so (once).  Raises ImportError when it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libispa.so not found at {LIB_PATH}; build it with "
                          "`python kv_cache_compression_two_b200/build.py` (needs nvcc)")
    L = ctypes.CDLL(LIB_PATH)
    sig = {
        "ispa_version": (ctypes.c_char_p, []),
        "ispa_last_error": (ctypes.c_char_p, []),
        "ispa_launch_count": (ctypes.c_uint64, []),
        "ispa_check_device_error": (_ci, [_vp, ctypes.POINTER(_ci)]),
        "ispa_attn_split_workspace_bytes": (_sz, [ctypes.POINTER(AttnDesc)]),
        "ispa_attn_split": (_ci, [ctypes.POINTER(AttnDesc)] + [_vp] * 10 + [_sz, _vp]),
        "ispa_lse_merge": (_ci, [_ci, _ci, _ci, _ci, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
        "ispa_accum_stats_workspace_bytes": (_sz, [_ci, _ci, _ci, _ci]),
        "ispa_accum_stats": (_ci, [_ci, _ci, _ci, _vp, _vp, _vp, _vp, _vp, _vp, _ci, _vp, _sz, _vp]),
        "ispa_ridge_workspace_bytes": (_sz, [_ci, _ci]),
        "ispa_ridge_solve": (_ci, [_ci, _ci, _vp, _vp, _vp, _cf, _ci, _ci, _vp, _vp, _vp, _sz, _vp]),
        "ispa_ridge_solve_noalloc": (_ci, [_ci, _ci, _vp, _vp, _vp, _cf, _ci, _ci, _vp, _vp, _vp]),
        "ispa_select_layers": (_ci, [_ci, _vp, _ci, _vp, _vp, _vp]),
        "ispa_absorb_weight": (_ci, [_ci, _ci, _vp, _ci, _vp, _vp, _ci, _vp]),
        "ispa_attn_local_proj_workspace_bytes": (_sz, [ctypes.POINTER(AttnDesc)]),
        "ispa_attn_local_proj": (_ci, [ctypes.POINTER(AttnDesc), _vp, _vp, _vp, _vp, _ci, _vp, _ci, _vp, _sz, _vp]),
        "ispa_kv_evicted_desc": (_ci, [ctypes.POINTER(AttnDesc), ctypes.POINTER(AttnDesc)]),
        "ispa_kv_evict_history": (_ci, [ctypes.POINTER(AttnDesc), _vp, _vp, _vp, _vp, _vp]),
        "ispa_kv_restore": (_ci, [ctypes.POINTER(AttnDesc), _vp, _vp, _vp, _vp, _vp]),
        "ispa_stats_reset": (_ci, [_ci, _ci, _vp, _vp, _vp, _vp]),
        "ispa_selftest_wait_timeout": (_ci, [ctypes.c_longlong, _vp]),
        "ispa_quantize_rows": (_ci, [_ci, _ci, _vp, _ci, _vp, _vp, _vp]),
        "ispa_quantize_weight": (_ci, [_ci, _ci, _vp, _ci, _vp, _vp, _vp]),
        "ispa_gemm_q8": (_ci, [_ci, _ci, _ci, _vp, _vp, _vp, _vp, _ci, _vp, _ci, _vp]),
        "ispa_gemm_bf16": (_ci, [_ci, _ci, _ci, _vp, _vp, _vp, _ci, _vp]),
        "ispa_attn_local_proj_q8_workspace_bytes": (_sz, [ctypes.POINTER(AttnDesc)]),
        "ispa_warmup_fused_workspace_bytes": (_sz, [ctypes.POINTER(AttnDesc), _ci]),
        "ispa_warmup_fused": (_ci, [ctypes.POINTER(AttnDesc), _vp, _vp, _vp, _vp, _ci, _vp, _vp, _vp, _vp, _vp, _vp,
                                    _sz, _vp]),
        "ispa_attn_local_proj_q8": (_ci, [ctypes.POINTER(AttnDesc), _vp, _vp, _vp, _vp, _vp, _ci, _ci, _vp, _ci,
                                          _vp, _sz, _vp]),
        "ispa_v16_bytes": (_sz, [ctypes.POINTER(AttnDesc)]),
        "ispa_absorb_error_workspace_bytes": (_sz, [_ci, _ci]),
        "ispa_kv8_bytes": (_sz, [ctypes.POINTER(AttnDesc)]),
        "ispa_kv8_prepare": (_ci, [ctypes.POINTER(AttnDesc), _vp, _vp, _ci, _ci, _vp, _vp]),
        "ispa_absorb_error": (_ci, [_ci, _ci, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
        "ispa_v16_prepare": (_ci, [ctypes.POINTER(AttnDesc), _vp, _ci, _ci, _vp, _vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _ptr(x, *, dtype=None, name="tensor") -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    import torch
    if not isinstance(x, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, an int address or None")
    if not x.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if not x.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if dtype is not None and x.dtype not in dtype:
        raise ValueError(f"{name}: dtype {x.dtype} not in {dtype}")
    return x.data_ptr()


def _stream(s) -> Optional[int]:
    if s is None:
        try:
            import torch
            if torch.cuda.is_available() and torch.cuda.is_initialized():
                return torch.cuda.current_stream().cuda_stream
        except Exception:
            pass
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(status: int) -> None:
    if status != ISPA_OK:
        raise IspaError(status, lib().ispa_last_error().decode(errors="replace"))


def _dt(t) -> int:
    import torch
    return ISPA_BF16 if t.dtype == torch.bfloat16 else ISPA_F32


def version() -> str:
    return lib().ispa_version().decode()


def launch_count() -> int:
    """Kernels enqueued by libispa so far in this process."""
    return int(lib().ispa_launch_count())


def ispa_check_device_error(stream=None) -> int:
    detail = ctypes.c_int(0)
    _check(lib().ispa_check_device_error(_stream(stream), ctypes.byref(detail)))
    return detail.value


def _ws(workspace, workspace_bytes):
    if workspace is not None and not isinstance(workspace, int):
        return _ptr(workspace, name="workspace"), workspace_bytes or workspace.numel() * workspace.element_size()
    return workspace, workspace_bytes


def ispa_attn_split_workspace_bytes(desc: AttnDesc) -> int:
    return int(lib().ispa_attn_split_workspace_bytes(ctypes.byref(desc)))


def ispa_attn_split(desc: AttnDesc, q, k, v, o_loc, lse_loc, o_hist=None, lse_hist=None, o_full=None, lse_full=None,
                    workspace=None, workspace_bytes: int = 0, stream=None) -> None:
    ws, nbytes = _ws(workspace, workspace_bytes)
    _check(lib().ispa_attn_split(ctypes.byref(desc), _ptr(q, name="q"), _ptr(k, name="k"), _ptr(v, name="v"),
                                 _ptr(o_loc, name="o_loc"), _ptr(lse_loc, name="lse_loc"), _ptr(o_hist, name="o_hist"),
                                 _ptr(lse_hist, name="lse_hist"), _ptr(o_full, name="o_full"),
                                 _ptr(lse_full, name="lse_full"), ws, nbytes, _stream(stream)))


def ispa_v16_bytes(desc: AttnDesc) -> int:
    return int(lib().ispa_v16_bytes(ctypes.byref(desc)))


def ispa_v16_prepare(desc: AttnDesc, v, frame_begin: int, frame_end: int, v16, stream=None) -> None:
    _check(lib().ispa_v16_prepare(ctypes.byref(desc), _ptr(v, name="v"), frame_begin, frame_end,
                                  _ptr(v16, name="v16"), _stream(stream)))


def ispa_kv8_bytes(desc: AttnDesc) -> int:
    return int(lib().ispa_kv8_bytes(ctypes.byref(desc)))


def ispa_kv8_prepare(desc: AttnDesc, k, v, frame_begin: int, frame_end: int, kv8, stream=None) -> None:
    _check(lib().ispa_kv8_prepare(ctypes.byref(desc), _ptr(k, name="k"), _ptr(v, name="v"), frame_begin, frame_end,
                                  _ptr(kv8, name="kv8"), _stream(stream)))


def ispa_lse_merge(rows: int, H: int, head_dim: int, o_dtype: int, o_a, lse_a, o_b, lse_b, o_out, lse_out,
                   stream=None) -> None:
    _check(lib().ispa_lse_merge(rows, H, head_dim, o_dtype, _ptr(o_a), _ptr(lse_a), _ptr(o_b), _ptr(lse_b),
                                _ptr(o_out), _ptr(lse_out), _stream(stream)))


def ispa_accum_stats_workspace_bytes(T: int, D: int, Dout: int, prec: int = ISPA_PREC_TF32) -> int:
    return int(lib().ispa_accum_stats_workspace_bytes(T, D, Dout, prec))


def ispa_accum_stats(T: int, D: int, Dout: int, a_loc, a_full, W, G, C, r2, prec: int = ISPA_PREC_TF32,
                     workspace=None, workspace_bytes: int = 0, stream=None) -> None:
    if workspace is not None and not isinstance(workspace, int):
        workspace_bytes = workspace_bytes or workspace.numel() * workspace.element_size()
    _check(lib().ispa_accum_stats(T, D, Dout, _ptr(a_loc), _ptr(a_full), _ptr(W), _ptr(G), _ptr(C), _ptr(r2), prec,
                                  _ptr(workspace), workspace_bytes, _stream(stream)))


def ispa_ridge_workspace_bytes(D: int, Dout: int) -> int:
    return int(lib().ispa_ridge_workspace_bytes(D, Dout))


def ispa_ridge_solve(D: int, Dout: int, G, C, r2, lam: float, lambda_relative: bool, refine_steps: int, dW, eps,
                     workspace, workspace_bytes: int = 0, stream=None) -> None:
    if workspace is not None and not isinstance(workspace, int):
        workspace_bytes = workspace_bytes or workspace.numel() * workspace.element_size()
    _check(lib().ispa_ridge_solve(D, Dout, _ptr(G), _ptr(C), _ptr(r2), float(lam), int(bool(lambda_relative)),
                                  int(refine_steps), _ptr(dW), _ptr(eps), _ptr(workspace), workspace_bytes,
                                  _stream(stream)))


def ispa_ridge_solve_noalloc(D: int, Dout: int, G, C, r2, lam: float, lambda_relative: bool, refine_steps: int, dW,
                             eps, stream=None) -> None:
    """ispa_ridge_solve without a workspace, for callers that cannot allocate device memory
    (D, Dout <= 1024; the scratch is a static array inside the library, shared by all calls)."""
    _check(lib().ispa_ridge_solve_noalloc(D, Dout, _ptr(G), _ptr(C), _ptr(r2), float(lam), int(bool(lambda_relative)),
                                          int(refine_steps), _ptr(dW), _ptr(eps), _stream(stream)))


def ispa_absorb_error_workspace_bytes(D: int, Dout: int) -> int:
    return int(lib().ispa_absorb_error_workspace_bytes(D, Dout))


def ispa_absorb_error(D: int, Dout: int, G, C, r2, dW, eps, workspace, workspace_bytes: int = 0,
                      stream=None) -> None:
    ws, nbytes = _ws(workspace, workspace_bytes)
    _check(lib().ispa_absorb_error(D, Dout, _ptr(G), _ptr(C), _ptr(r2), _ptr(dW), _ptr(eps), ws, nbytes,
                                   _stream(stream)))


def ispa_select_layers(N: int, eps, K: int, is_local, idx, stream=None) -> None:
    _check(lib().ispa_select_layers(N, _ptr(eps), K, _ptr(is_local), _ptr(idx), _stream(stream)))


def ispa_absorb_weight(D: int, Dout: int, W, w_dtype: int, dW, W_new, out_dtype: int, stream=None) -> None:
    _check(lib().ispa_absorb_weight(D, Dout, _ptr(W), w_dtype, _ptr(dW), _ptr(W_new), out_dtype, _stream(stream)))


def ispa_attn_local_proj_workspace_bytes(desc: AttnDesc) -> int:
    return int(lib().ispa_attn_local_proj_workspace_bytes(ctypes.byref(desc)))


def ispa_attn_local_proj(desc: AttnDesc, q, k, v, W_proj, Dout: int, y, y_dtype: int, workspace,
                         workspace_bytes: int = 0, stream=None) -> None:
    if workspace is not None and not isinstance(workspace, int):
        workspace_bytes = workspace_bytes or workspace.numel() * workspace.element_size()
    _check(lib().ispa_attn_local_proj(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(W_proj), Dout, _ptr(y),
                                      y_dtype, _ptr(workspace), workspace_bytes, _stream(stream)))


def ispa_quantize_rows(M: int, K: int, x, fmt: int, q, sa, stream=None) -> None:
    _check(lib().ispa_quantize_rows(M, K, _ptr(x), fmt, _ptr(q), _ptr(sa), _stream(stream)))


def ispa_quantize_weight(K: int, N: int, W, fmt: int, qT, sw, stream=None) -> None:
    _check(lib().ispa_quantize_weight(K, N, _ptr(W), fmt, _ptr(qT), _ptr(sw), _stream(stream)))


def ispa_gemm_q8(M: int, N: int, K: int, q, sa, qT, sw, fmt: int, y, y_dtype: int, stream=None) -> None:
    _check(lib().ispa_gemm_q8(M, N, K, _ptr(q), _ptr(sa), _ptr(qT), _ptr(sw), fmt, _ptr(y), y_dtype,
                              _stream(stream)))


def ispa_gemm_bf16(M: int, N: int, K: int, A, W, y, y_dtype: int, stream=None) -> None:
    _check(lib().ispa_gemm_bf16(M, N, K, _ptr(A), _ptr(W), _ptr(y), y_dtype, _stream(stream)))


def ispa_attn_local_proj_q8_workspace_bytes(desc: AttnDesc) -> int:
    return int(lib().ispa_attn_local_proj_q8_workspace_bytes(ctypes.byref(desc)))


def ispa_attn_local_proj_q8(desc: AttnDesc, q, k, v, qT, sw, fmt: int, Dout: int, y, y_dtype: int, workspace,
                            workspace_bytes: int = 0, stream=None) -> None:
    if workspace is not None and not isinstance(workspace, int):
        workspace_bytes = workspace_bytes or workspace.numel() * workspace.element_size()
    _check(lib().ispa_attn_local_proj_q8(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(qT), _ptr(sw), fmt,
                                         Dout, _ptr(y), y_dtype, _ptr(workspace), workspace_bytes,
                                         _stream(stream)))


def ispa_warmup_fused_workspace_bytes(desc: AttnDesc, Dout: int) -> int:
    return int(lib().ispa_warmup_fused_workspace_bytes(ctypes.byref(desc), Dout))


def ispa_warmup_fused(desc: AttnDesc, q, k, v, W, Dout: int, o_full, l_full, G, C, r2, workspace,
                      workspace_bytes: int = 0, stream=None) -> None:
    if workspace is not None and not isinstance(workspace, int):
        workspace_bytes = workspace_bytes or workspace.numel() * workspace.element_size()
    _check(lib().ispa_warmup_fused(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(W), Dout, _ptr(o_full),
                                   _ptr(l_full), _ptr(G), _ptr(C), _ptr(r2), _ptr(workspace), workspace_bytes,
                                   _stream(stream)))


def ispa_kv_evicted_desc(desc: AttnDesc) -> AttnDesc:
    out = AttnDesc()
    _check(lib().ispa_kv_evicted_desc(ctypes.byref(desc), ctypes.byref(out)))
    return out


def ispa_kv_evict_history(desc: AttnDesc, k, v, k_out, v_out, stream=None) -> None:
    _check(lib().ispa_kv_evict_history(ctypes.byref(desc), _ptr(k), _ptr(v), _ptr(k_out), _ptr(v_out),
                                       _stream(stream)))


def ispa_kv_restore(desc: AttnDesc, k_ev, v_ev, k_full, v_full, stream=None) -> None:
    _check(lib().ispa_kv_restore(ctypes.byref(desc), _ptr(k_ev), _ptr(v_ev), _ptr(k_full), _ptr(v_full),
                                 _stream(stream)))


def ispa_stats_reset(D: int, Dout: int, G, C, r2, stream=None) -> None:
    _check(lib().ispa_stats_reset(D, Dout, _ptr(G), _ptr(C), _ptr(r2), _stream(stream)))


ISPA_SELFTEST_SITE = 999


def ispa_selftest_wait_timeout(wait_ns: int, stream=None) -> None:
    _check(lib().ispa_selftest_wait_timeout(int(wait_ns), _stream(stream)))


lib()
