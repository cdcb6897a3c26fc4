"""The allocation-free ridge solve, against the oracle and the workspace form.

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

import numpy as np
import pytest
import torch

import kv_cache_compression_two_b200 as ispa
from oracle import ispa_oracle as orc

pytestmark = pytest.mark.gpu


def _problem(D, Dout, seed):
    g = np.random.default_rng(seed)
    A = g.standard_normal((3 * D, D))
    R = A @ g.standard_normal((D, Dout)) * 0.1 + 0.05 * g.standard_normal((3 * D, Dout))
    G = np.triu(A.T @ A).astype(np.float32)
    C = (A.T @ R).astype(np.float32)
    return G, C, float(np.sum(R * R))


def _noalloc(D, Dout, Gd, Cd, r2d, refine, dW, eps):
    """One call through the C ABI directly (no binding logic in between)."""
    st = ispa.lib().ispa_ridge_solve_noalloc(D, Dout, Gd.data_ptr(), Cd.data_ptr(), r2d.data_ptr(),
                                             ctypes.c_float(1e-4), 1, refine, dW.data_ptr(), eps.data_ptr(),
                                             torch.cuda.current_stream().cuda_stream)
    assert st == ispa.ISPA_OK, ispa.lib().ispa_last_error().decode()


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
    _noalloc(D, Dout, Gd, Cd, r2d, refine, dW_na, eps[1:2])
    ispa.ispa_check_device_error()
    return (G, C, r2, dW_ws.cpu().numpy().astype(np.float64), dW_na.cpu().numpy().astype(np.float64),
            eps.cpu().numpy())


def test_noalloc_matches_oracle_and_workspace_solve_on_two_calls_in_a_row():
    # two different problems back to back: the second call must not see the first call's scratch
    for D, Dout, seed, refine in ((512, 384, 1, 0), (1024, 1024, 2, 1)):
        G, C, r2, dW_ws, got, eps = _solve_both(D, Dout, seed, refine)
        assert np.all(np.isfinite(got))
        # against the fp64 oracle, with the ridge tests' tolerances: 1e-2 plain, 1e-5 refined
        Gs = np.triu(G).astype(np.float64)
        Gs = Gs + np.triu(Gs, 1).T
        lam32 = float(np.float32(orc.ridge_lambda(Gs, 1e-4, True)))
        ref = orc.ridge_solve(Gs, C.astype(np.float64), lam32)
        tol = 1e-5 if refine else 1e-2
        err = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        assert err <= tol, err
        # epsilon against the oracle's at its own dW*: the quadratic form moves by at most
        # 2 lam tol |dW*|^2 + |G|_2 tol^2 |dW*|^2, plus 1e-6 r2 for the kernel's rounding
        ref_eps = orc.eps_from_stats(Gs, C.astype(np.float64), r2, ref)
        n2 = float(np.sum(ref * ref))
        bound = 1e-6 * r2 + 2.0 * lam32 * tol * n2 + float(np.abs(Gs).sum(axis=1).max()) * tol ** 2 * n2
        assert abs(eps[1] - ref_eps) <= bound, (eps[1], ref_eps, bound)
        # and the same arithmetic as the workspace form (the scratch layout is the workspace's;
        # the two differ only by the order of the solve products' atomic additions), epsilon
        # within the quadratic form's bound for that difference
        rho = np.linalg.norm(got - dW_ws) / np.linalg.norm(dW_ws)
        assert rho <= 1e-6, rho
        n2w = float(np.sum(dW_ws * dW_ws))
        assert abs(eps[1] - eps[0]) <= 1e-6 * r2 + 2.0 * lam32 * rho * n2w + float(np.abs(Gs).sum(axis=1).max()) * rho ** 2 * n2w


def test_noalloc_allocates_no_device_memory():
    D = Dout = 256
    G, C, r2 = _problem(D, Dout, 3)
    Gd, Cd = torch.from_numpy(G).cuda(), torch.from_numpy(C).cuda()
    r2d = torch.tensor([r2], dtype=torch.float64, device="cuda")
    dW = torch.empty((D, Dout), device="cuda")
    eps = torch.zeros(1, dtype=torch.float64, device="cuda")
    _noalloc(D, Dout, Gd, Cd, r2d, 0, dW, eps)   # warm-up: loads the module and looks up the array
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    for refine in (0, 2):
        _noalloc(D, Dout, Gd, Cd, r2d, refine, dW, eps)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 == free0, (free0, free1)
    assert ispa.ispa_check_device_error() == ispa.ISPA_OK


def test_noalloc_rejects_sizes_beyond_its_scratch():
    D = ispa.RIDGE_NOALLOC_MAX_D + 1
    st = ispa.lib().ispa_ridge_solve_noalloc(D, 64, 0x10000, 0x10000, 0x10000, ctypes.c_float(0.0), 0, 0, 0x10000,
                                             0x10000, None)
    assert st == ispa.ISPA_ERR_INVALID_ARG
    msg = ispa.lib().ispa_last_error().decode()
    assert "1024" in msg and "workspace" in msg
