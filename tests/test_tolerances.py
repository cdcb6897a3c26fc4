"""CPU checks of the arithmetic behind the GPU parity bounds.

The fp8 attention tests treat weights that lie within a relative 2^-14 of an
e4m3 rounding boundary as ties (either neighbouring code is a correct result
at the kernel's precision).  That figure rests on how far the kernel's fp32
weights can sit from the oracle's fp64 ones; this file models the kernel's
fp32 arithmetic on the test layouts' data and checks the distance.
"""
import math

import numpy as np

from oracle import ispa_oracle as orc
import synth_inputs as si

TIE_REL = 2.0 ** -14


def _f32_toward_zero(x: np.ndarray) -> np.ndarray:
    """fp64 values rounded to fp32 toward zero (the tensor cores' accumulation)."""
    r = x.astype(np.float32)
    over = np.abs(r.astype(np.float64)) > np.abs(x)
    r[over] = np.nextafter(r[over], np.float32(0.0))
    return r


def _scores_f32(q8: np.ndarray, k8: np.ndarray) -> np.ndarray:
    """q8 k8^T over d = 128 as four products of K = 32, each block's sum taken
    exactly (e4m3 products are exact in fp32) and rounded to fp32, the blocks
    accumulated in fp32 rounding toward zero."""
    acc = np.zeros((q8.shape[0], k8.shape[0]), np.float32)
    for kk in range(0, q8.shape[1], 32):
        part = (q8[:, kk:kk + 32] @ k8[:, kk:kk + 32].T).astype(np.float32)
        acc = _f32_toward_zero(acc.astype(np.float64) + part.astype(np.float64))
    return acc


def test_fp8_kernel_weights_stay_within_the_tie_tolerance_of_the_oracle():
    """Scores in fp32 as above, t = S c with c = s_q s_k scale log2(e) in fp32, the
    block maximum and x = S c + (6 - m) in fp32; the weight 2^x against the oracle's
    2^(t - m + 6) in fp64: relative distance below TIE_REL / 4 on iid heads and on
    heads scaled by 2^10 (Q) and 2^-12 (K), whose scores reach tens of log2 units."""
    sh = si.AttnShape(B=1, H=2, d=128, tpf=50, sink_frames=2, hist_begin=2, hist_end=7, cur_begin=7, cur_end=10,
                      kv_frames=10)
    worst = 0.0
    for key, qs, ks in ((("tol", "iid"), 1.0, 1.0), (("tol", "scaled"), 2.0 ** 10, 2.0 ** -12),
                        (("tol", "peaked"), 8.0, 4.0)):
        data = si.iid_qkv(sh, "bf16", key)
        q = si.round_to_bf16(data["q"] * np.float32(qs))
        k = si.round_to_bf16(data["k"] * np.float32(ks))
        q8, sq = orc.quantize_heads(q)
        k8, sk = orc.quantize_heads(k)
        for h in range(sh.H):
            c64 = float(sq[0, h]) * float(sk[0, h]) / math.sqrt(sh.d) / math.log(2.0)
            c32 = np.float32(np.float32(sq[0, h]) * np.float32(sk[0, h])) * \
                np.float32(1.0 / math.sqrt(sh.d) * 1.4426950408889634)
            t64 = (q8[0, :, h, :] @ k8[0, :, h, :].T) * c64
            s32 = _scores_f32(q8[0, :, h, :], k8[0, :, h, :])
            for lo in range(0, t64.shape[1], 128):
                tb = t64[:, lo:lo + 128]
                sb = s32[:, lo:lo + 128]
                m64 = tb.max(axis=1, keepdims=True)
                m32 = (sb.max(axis=1, keepdims=True) * c32).astype(np.float32)
                x32 = (sb.astype(np.float64) * float(c32) + (np.float32(6.0) - m32).astype(np.float64))
                x32 = x32.astype(np.float32).astype(np.float64)  # the fused multiply-add's one rounding
                x64 = tb - m64 + 6.0
                keep = x64 > -20.0  # weights that reach the e4m3 grid at all
                rel = np.abs(np.exp2(x32[keep] - x64[keep]) - 1.0)
                worst = max(worst, float(rel.max()))
    assert worst < TIE_REL / 4, worst


def test_bf16_projection_error_model_sits_well_inside_its_bound():
    """The post-switch projection y = A_loc (W + dW) runs in bf16 (both operands
    rounded to bf16, fp32 accumulation); its parity bound is 2e-2 of the output's
    RMS.  Modelled on the CPU at the tests' shapes -- A_loc unit-scale like an
    attention output, W a projection weight -- the largest deviation from the
    fp64 product stays under half the bound."""
    g = si.rng("tol", "proj")
    for T, D, Dout in ((405, 256, 192), (780, 1536, 1536)):
        A = g.standard_normal((T, D)) * 0.5
        W = si.projection_weight(D, Dout, ("tol", "proj", D), "bf16").astype(np.float64)
        dW = 0.02 * g.standard_normal((D, Dout))
        Wn = si.round_to_bf16((W + dW).astype(np.float32)).astype(np.float64)
        exact = A @ Wn
        model = (si.round_to_bf16(A.astype(np.float32)).astype(np.float32) @ Wn.astype(np.float32)).astype(np.float64)
        rel = np.abs(model - exact).max() / np.sqrt(np.mean(exact ** 2))
        assert rel < 1e-2, (T, D, rel)
