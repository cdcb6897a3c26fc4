"""The allocation-free ridge solve against the workspace form.

ispa_ridge_solve_noalloc serves callers that cannot allocate device memory
for a workspace: a generator's per-chunk loop that must not call cudaMalloc
or cudaFree (they can synchronise the device and stall the streams still
producing frames), or a host whose device memory belongs to another
allocator.  Its scratch is a static array inside the library shared by all
calls.  This file is named so that pytest collects it last; it sets up
everything it needs itself and passes both alone in a fresh process and after
the other tests.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import kv_cache_compression_two_b200 as ispa

pytestmark = pytest.mark.gpu


def _problem(D, Dout, seed):
    g = np.random.default_rng(seed)
    A = g.standard_normal((3 * D, D))
    R = A @ g.standard_normal((D, Dout)) * 0.1 + 0.05 * g.standard_normal((3 * D, Dout))
    G = np.triu(A.T @ A).astype(np.float32)
    C = (A.T @ R).astype(np.float32)
    return G, C, float(np.sum(R * R))


def _solve_both(D, Dout, seed, refine):
    G, C, r2 = _problem(D, Dout, seed)
    Gd = torch.from_numpy(G).cuda()
    Cd = torch.from_numpy(C).cuda()
    r2d = torch.tensor([r2], dtype=torch.float64, device="cuda")
    dW_ws = torch.full((D, Dout), float("nan"), device="cuda")
    dW_na = torch.full((D, Dout), float("nan"), device="cuda")
    eps = torch.zeros(2, dtype=torch.float64, device="cuda")
    ws = torch.empty(ispa.ispa_ridge_workspace_bytes(D, Dout), dtype=torch.uint8, device="cuda")
    ispa.ispa_ridge_solve(D, Dout, Gd, Cd, r2d, 1e-4, True, refine, dW_ws, eps[0:1], ws)
    # through the C ABI directly
    st = ispa.lib().ispa_ridge_solve_noalloc(D, Dout, Gd.data_ptr(), Cd.data_ptr(), r2d.data_ptr(),
                                             ctypes.c_float(1e-4), 1, refine, dW_na.data_ptr(),
                                             eps[1:2].data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == ispa.ISPA_OK, ispa.lib().ispa_last_error().decode()
    ispa.ispa_check_device_error()
    return dW_ws.cpu().numpy().astype(np.float64), dW_na.cpu().numpy().astype(np.float64), eps.cpu().numpy(), r2


def test_noalloc_matches_workspace_solve_on_two_calls_in_a_row():
    # two different problems back to back: the second call must not see the first call's scratch
    for D, Dout, seed, refine in ((512, 384, 1, 0), (1024, 1024, 2, 1)):
        ref, got, eps, r2 = _solve_both(D, Dout, seed, refine)
        assert np.all(np.isfinite(got))
        err = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        assert err <= 1e-2, err                       # the dW tolerance of the ridge tests
        assert abs(eps[1] - eps[0]) <= 1e-6 * r2      # the epsilon tolerance of the ridge tests


def test_noalloc_rejects_sizes_beyond_its_scratch():
    D = ispa.RIDGE_NOALLOC_MAX_D + 1
    st = ispa.lib().ispa_ridge_solve_noalloc(D, 64, 0x10000, 0x10000, 0x10000, ctypes.c_float(0.0), 0, 0, 0x10000,
                                             0x10000, None)
    assert st == ispa.ISPA_ERR_INVALID_ARG
    msg = ispa.lib().ispa_last_error().decode()
    assert "1024" in msg and "workspace" in msg
