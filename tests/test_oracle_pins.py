"""Pins of the fp64 oracle to facts fixed by the ISPA pages and by mathematics.

No test here compares the oracle with itself: each one checks it against a
brute-force computation written independently (pure-Python loops), a closed
form, an invariant, a LAPACK/NumPy routine solving the same problem another
way, or a value printed on the pages.  The mutation tests at the end plant a
plausible mistake in a copy of an oracle function and check that a pin
catches it.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

from oracle import ispa_oracle as orc
import synth_inputs as si

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------
# brute-force softmax attention, independent of the oracle (pure Python)
# ---------------------------------------------------------------------------
def brute_attention(q, k, v, scale):
    """Softmax attention of each query over all rows of k/v, with math.exp loops."""
    n, d = len(q), len(q[0])
    O = np.zeros((n, len(v[0]) if len(v) else d))
    L = np.zeros(n)
    for i in range(n):
        s = [scale * sum(float(q[i][t]) * float(kj[t]) for t in range(d)) for kj in k]
        if not s:
            O[i] = 0.0
            L[i] = -math.inf
            continue
        mx = max(s)
        w = [math.exp(x - mx) for x in s]
        tot = math.fsum(w)
        for j, wj in enumerate(w):
            O[i] += (wj / tot) * np.asarray(v[j], np.float64)
        L[i] = mx + math.log(tot)
    return O, L


def _rand(g, *shape, std=1.0):
    return g.standard_normal(shape) * std


# ---------------------------------------------------------------------------
# P1: per-group attention and the merge equal monolithic softmax
# ---------------------------------------------------------------------------
def check_group_vs_brute(attend, seed=0):
    g = np.random.default_rng(seed)
    ok = True
    for n, m, d in [(3, 5, 4), (1, 1, 2), (4, 9, 8)]:
        q, k, v = _rand(g, n, d), _rand(g, m, d), _rand(g, m, d)
        scale = 1.0 / math.sqrt(d)
        O, L = attend(q, k, v, scale)
        Ob, Lb = brute_attention(q, k, v, scale)
        ok &= np.allclose(O, Ob, rtol=1e-12, atol=1e-13) and np.allclose(L, Lb, rtol=1e-13, atol=1e-13)
    return bool(ok)


def test_group_attention_bruteforce():
    assert check_group_vs_brute(orc.attend_group)


def test_group_attention_closed_forms():
    g = np.random.default_rng(1)
    d, m = 8, 7
    q = _rand(g, 3, d)
    kvec = _rand(g, d)
    k = np.tile(kvec, (m, 1))              # identical keys -> uniform weights
    v = _rand(g, m, d)
    O, L = orc.attend_group(q, k, v, 0.5)
    s = 0.5 * (q @ kvec)
    assert np.allclose(O, np.tile(v.mean(axis=0), (3, 1)), atol=1e-14)
    assert np.allclose(L, s + math.log(m), atol=1e-13)
    O1, L1 = orc.attend_group(q, k[:1], v[:1], 0.5)   # single key -> O = v, L = s
    assert np.allclose(O1, np.tile(v[0], (3, 1)), atol=1e-15)
    assert np.allclose(L1, s, atol=1e-15)
    O0, L0 = orc.attend_group(q, k[:0], v[:0], 0.5)   # empty group
    assert np.all(O0 == 0) and np.all(np.isneginf(L0))


def check_merge_vs_monolithic(merge, seed=2):
    """Random two-way splits of a key set: merged (O, L) == attention over the union."""
    g = np.random.default_rng(seed)
    ok = True
    for trial in range(40):
        d = int(g.choice([2, 4, 8]))
        n, m = int(g.integers(1, 5)), int(g.integers(1, 40))
        mult = [1.0, 30.0][trial % 2]      # x30 scores stress overflow handling
        q, k, v = _rand(g, n, d) * mult, _rand(g, m, d), _rand(g, m, d)
        perm = g.permutation(m)
        cut = int(g.integers(0, m + 1))    # cut == 0 or m leaves one group empty
        a, b = perm[:cut], perm[cut:]
        oa, la = orc.attend_group(q, k[a], v[a], 0.3)
        ob, lb = orc.attend_group(q, k[b], v[b], 0.3)
        O, L = merge(oa, la, ob, lb)
        Ob, Lb = brute_attention(q, k, v, 0.3)
        ok &= np.allclose(O, Ob, rtol=1e-10, atol=1e-12) and np.allclose(L, Lb, rtol=1e-12, atol=1e-10)
    return bool(ok)


def test_merge_equals_monolithic_softmax():
    assert check_merge_vs_monolithic(orc.lse_merge)


def test_merge_dominant_history_and_empty_groups():
    g = np.random.default_rng(3)
    d = 4
    q = _rand(g, 2, d)
    k_loc, v_loc = _rand(g, 3, d), _rand(g, 3, d)
    # history keys aligned with q and scaled so its LSE exceeds the local one by > 50 nats
    k_hist = np.stack([q[0] * 60.0, q[1] * 60.0])
    v_hist = _rand(g, 2, d)
    ol, ll = orc.attend_group(q, k_loc, v_loc, 1.0)
    oh, lh = orc.attend_group(q, k_hist, v_hist, 1.0)
    assert np.all(lh - ll > 50)
    O, L = orc.lse_merge(ol, ll, oh, lh)
    Ob, Lb = brute_attention(q, np.vstack([k_loc, k_hist]), np.vstack([v_loc, v_hist]), 1.0)
    assert np.allclose(O, Ob, atol=1e-12) and np.allclose(L, Lb, atol=1e-9)
    # empty history: full == local exactly
    e_o, e_l = np.zeros_like(ol), np.full(2, -np.inf)
    O2, L2 = orc.lse_merge(ol, ll, e_o, e_l)
    assert np.array_equal(O2, ol) and np.array_equal(L2, ll)
    # both empty
    O3, L3 = orc.lse_merge(e_o, e_l, e_o, e_l)
    assert np.all(O3 == 0) and np.all(np.isneginf(L3))


# ---------------------------------------------------------------------------
# P2: merge symmetry and associativity
# ---------------------------------------------------------------------------
def test_merge_symmetry_and_associativity():
    g = np.random.default_rng(4)
    d, n = 8, 5
    q = _rand(g, n, d)
    groups = [(_rand(g, m, d), _rand(g, m, d)) for m in (3, 7, 11)]
    parts = [orc.attend_group(q, k, v, 0.4) for k, v in groups]
    ab = orc.lse_merge(*parts[0], *parts[1])
    ba = orc.lse_merge(*parts[1], *parts[0])
    assert np.allclose(ab[0], ba[0], atol=1e-15) and np.allclose(ab[1], ba[1], atol=1e-15)
    left = orc.lse_merge(*ab, *parts[2])
    bc = orc.lse_merge(*parts[1], *parts[2])
    right = orc.lse_merge(*parts[0], *bc)
    assert np.allclose(left[0], right[0], atol=1e-14) and np.allclose(left[1], right[1], atol=1e-13)
    kall = np.vstack([k for k, _ in groups])
    vall = np.vstack([v for _, v in groups])
    Ob, Lb = brute_attention(q, kall, vall, 0.4)
    assert np.allclose(left[0], Ob, atol=1e-12) and np.allclose(left[1], Lb, atol=1e-12)


# ---------------------------------------------------------------------------
# split attention over frame layouts: groups partition the KV (no frame twice)
# ---------------------------------------------------------------------------
def test_split_attention_layouts_bruteforce():
    g = np.random.default_rng(5)
    shapes = [si.random_groups_shape(g, max_frames=4, d=4, H=2, tpf=3, B=1) for _ in range(6)]
    # first chunk of a video: the current chunk is the sink itself (union, no double count)
    shapes.append(si.AttnShape(B=1, H=1, d=4, tpf=2, sink_frames=2, hist_begin=2, hist_end=2,
                               cur_begin=0, cur_end=2, kv_frames=2))
    # sink overlapping part of the current chunk
    shapes.append(si.AttnShape(B=1, H=1, d=4, tpf=2, sink_frames=2, hist_begin=2, hist_end=2,
                               cur_begin=1, cur_end=3, kv_frames=3))
    for sh in shapes:
        q = _rand(g, sh.B, sh.Lq, sh.H, sh.d)
        k = _rand(g, sh.B, sh.Lkv, sh.H, sh.d)
        v = _rand(g, sh.B, sh.Lkv, sh.H, sh.d)
        out = orc.split_attention(sh, q, k, v)
        frames_loc = sorted(set(range(sh.sink_frames)) | set(range(sh.cur_begin, sh.cur_end)))
        rows_loc = [f * sh.tpf + t for f in frames_loc for t in range(sh.tpf)]
        rows_hist = list(range(sh.hist_begin * sh.tpf, sh.hist_end * sh.tpf))
        assert not set(rows_loc) & set(rows_hist)
        for h in range(sh.H):
            sc = 1.0 / math.sqrt(sh.d)
            Ol, Ll = brute_attention(q[0, :, h], k[0, rows_loc, h], v[0, rows_loc, h], sc)
            Of, Lf = brute_attention(q[0, :, h], k[0, rows_loc + rows_hist, h], v[0, rows_loc + rows_hist, h], sc)
            assert np.allclose(out["O_loc"][0, :, h], Ol, atol=1e-12)
            assert np.allclose(out["L_loc"][0, :, h], Ll, atol=1e-12)
            assert np.allclose(out["O_full"][0, :, h], Of, atol=1e-12)
            assert np.allclose(out["L_full"][0, :, h], Lf, atol=1e-12)
        if sh.hist_end == sh.hist_begin:
            assert np.all(np.isneginf(out["L_hist"])) and np.all(out["O_hist"] == 0)


def test_full_attention_is_merge_of_groups():
    sh = si.TINY
    d = si.iid_qkv(sh, "f32", ("pin", "full"))
    out = orc.split_attention(sh, d["q"], d["k"], d["v"])
    O, L = orc.full_attention(sh, d["q"], d["k"], d["v"])
    assert np.allclose(out["O_full"], O, atol=1e-13) and np.allclose(out["L_full"], L, atol=1e-12)


# ---------------------------------------------------------------------------
# P3: exact absorption; P4: normal equations; P5: library cross-checks
# ---------------------------------------------------------------------------
def _absorb_problem(seed, T=200, D=12, Dout=10):
    g = np.random.default_rng(seed)
    A_loc = _rand(g, T, D)
    A_full = A_loc + 0.3 * _rand(g, T, D)
    W = _rand(g, D, Dout) / math.sqrt(D)
    return A_loc, A_full, W


def check_exact_absorption(stats, solve, eps_fn, seed=6):
    g = np.random.default_rng(seed)
    T, D, Dout = 60, 8, 6
    A_loc = _rand(g, T, D)
    M = np.eye(D) + 0.4 * _rand(g, D, D)
    A_full = A_loc @ M
    W = _rand(g, D, Dout)
    G, C, r2 = stats(A_loc, A_full, W)
    dW = solve(G, C, 0.0)
    e = eps_fn(A_loc, A_full, W, dW)
    return bool(np.allclose(dW, (M - np.eye(D)) @ W, atol=1e-10) and e <= 1e-20 * r2 + 1e-24)


def test_exact_absorption_closed_form():
    assert check_exact_absorption(orc.absorption_stats, orc.ridge_solve, orc.eps_direct)


def test_absorb_layer_stacks_every_chunk_and_absorbs_exactly():
    """Three warmup chunks of a layer (two instances, two heads of d = 4) whose full
    output is an exact linear map of the local one, A_full = A_loc M: with lambda -> 0
    the layer's absorption is dW = (M - I) W and eps = 0; its statistics are the sums
    of the chunks' own (explicit loops over every row of every chunk); the relative
    lambda takes the trace of the summed G; and the history output plays no part."""
    g = np.random.default_rng(21)
    B, n, H, d = 2, 7, 2, 4
    D = H * d
    M = np.eye(D) + 0.3 * g.standard_normal((D, D))
    W = g.standard_normal((D, 5))
    chunks = []
    for _ in range(3):
        o_loc = g.standard_normal((B, n, H, d))
        o_full = (o_loc.reshape(B * n, D) @ M).reshape(B, n, H, d)
        chunks.append({"O_loc": o_loc, "O_full": o_full, "O_hist": np.full((B, n, H, d), np.nan)})
    out = orc.absorb_layer(chunks, W, 1e-14, False)
    assert np.allclose(out["dW"], (M - np.eye(D)) @ W, atol=1e-8)
    assert out["eps"] <= 1e-12 * out["r2"]
    G = np.zeros((D, D))
    C = np.zeros((D, 5))
    r2 = 0.0
    for c in chunks:
        for b in range(B):
            for i in range(n):
                a = [c["O_loc"][b, i, h, e] for h in range(H) for e in range(d)]
                f = [c["O_full"][b, i, h, e] for h in range(H) for e in range(d)]
                r = [sum((f[k] - a[k]) * W[k, j] for k in range(D)) for j in range(5)]
                for x in range(D):
                    for y in range(D):
                        G[x, y] += a[x] * a[y]
                    for j in range(5):
                        C[x, j] += a[x] * r[j]
                r2 += sum(v * v for v in r)
    assert np.allclose(out["G"], G, rtol=1e-12, atol=1e-12) and np.allclose(out["C"], C, rtol=1e-12, atol=1e-12)
    assert abs(out["r2"] - r2) <= 1e-12 * r2
    rel = orc.absorb_layer(chunks, W, 1e-3, True)
    assert abs(rel["lam"] - 1e-3 * np.trace(G) / D) <= 1e-12 * rel["lam"]


def check_normal_equations(stats, solve, lam=0.7, seed=7):
    A_loc, A_full, W = _absorb_problem(seed)
    G, C, r2 = stats(A_loc, A_full, W)
    dW = solve(G, C, lam)
    R = (A_full - A_loc) @ W
    resid = A_loc.T @ (A_loc @ dW - R) + lam * dW
    return bool(np.abs(resid).max() <= 1e-9 * np.abs(A_loc.T @ R).max())


def test_normal_equations():
    assert check_normal_equations(orc.absorption_stats, orc.ridge_solve, lam=0.7)
    assert check_normal_equations(orc.absorption_stats, orc.ridge_solve, lam=0.0)


def test_ridge_against_lstsq_and_svd_filter():
    A_loc, A_full, W = _absorb_problem(8)
    G, C, r2 = orc.absorption_stats(A_loc, A_full, W)
    R = (A_full - A_loc) @ W
    dW0 = orc.ridge_solve(G, C, 0.0)
    ls = np.linalg.lstsq(A_loc, R, rcond=None)[0]
    assert np.allclose(dW0, ls, atol=1e-10)
    lam = 3.0
    U, s, Vt = np.linalg.svd(A_loc, full_matrices=False)
    svd_sol = Vt.T @ np.diag(s / (s ** 2 + lam)) @ U.T @ R
    assert np.allclose(orc.ridge_solve(G, C, lam), svd_sol, atol=1e-11)
    big = orc.ridge_solve(G, C, 1e12)
    assert np.abs(big).max() < 1e-8
    assert orc.eps_direct(A_loc, A_full, W, big) == pytest.approx(r2, rel=1e-6)


def test_stats_are_the_gram_and_cross_products():
    # G and C written as explicit row sums (sum_t a_t a_t^T) in Python loops
    A_loc, A_full, W = _absorb_problem(9, T=15, D=4, Dout=3)
    G, C, r2 = orc.absorption_stats(A_loc, A_full, W)
    Gb = np.zeros((4, 4)); Cb = np.zeros((4, 3)); r2b = 0.0
    for t in range(15):
        a = A_loc[t]
        r = [sum((A_full[t, i] - A_loc[t, i]) * W[i, j] for i in range(4)) for j in range(3)]
        for i in range(4):
            for j in range(4):
                Gb[i, j] += a[i] * a[j]
            for j in range(3):
                Cb[i, j] += a[i] * r[j]
        r2b += sum(x * x for x in r)
    assert np.allclose(G, Gb, atol=1e-12) and np.allclose(C, Cb, atol=1e-12)
    assert r2 == pytest.approx(r2b, rel=1e-13)


def test_cholesky_factor():
    g = np.random.default_rng(10)
    X = _rand(g, 30, 9)
    A = X.T @ X + 0.1 * np.eye(9)
    L = orc.cholesky_lower(A)
    assert np.allclose(np.triu(L, 1), 0) and np.all(np.diag(L) > 0)
    assert np.allclose(L @ L.T, A, atol=1e-12)


def test_relative_lambda():
    G = np.diag([1.0, 2.0, 3.0, 6.0])
    assert orc.ridge_lambda(G, 1e-4, True) == pytest.approx(1e-4 * 12.0 / 4)
    assert orc.ridge_lambda(G, 1e-3, False) == 1e-3


# ---------------------------------------------------------------------------
# P9: epsilon two ways
# ---------------------------------------------------------------------------
def test_eps_direct_equals_stats_form():
    for seed, lam in [(11, 0.0), (12, 0.5), (13, 50.0)]:
        A_loc, A_full, W = _absorb_problem(seed)
        G, C, r2 = orc.absorption_stats(A_loc, A_full, W)
        dW = orc.ridge_solve(G, C, lam)
        e1 = orc.eps_direct(A_loc, A_full, W, dW)
        e2 = orc.eps_from_stats(G, C, r2, dW)
        assert e1 == pytest.approx(e2, rel=1e-10, abs=1e-10 * r2)
        # the ridge solution never does worse than no correction
        assert e1 <= r2 * (1 + 1e-12)


# ---------------------------------------------------------------------------
# P6: selection == brute force over subsets
# ---------------------------------------------------------------------------
def check_selection_bruteforce(select, seed=14):
    g = np.random.default_rng(seed)
    ok = True
    for N in range(1, 9):
        for _ in range(5):
            eps = np.round(g.random(N) * 4) / 4         # frequent ties
            for K in range(0, N + 1):
                mask, idx = select(eps, K)
                combos = list(itertools.combinations(range(N), K))
                best_sum = min(float(np.sum(eps[list(c)])) for c in combos)
                # minimal total epsilon; among equal totals the lower layer indices win
                expected = min(c for c in combos if float(np.sum(eps[list(c)])) == best_sum)
                ok &= list(idx) == list(expected) and int(mask.sum()) == K and all(mask[list(idx)] == 1)
    return bool(ok)


def test_selection_bruteforce():
    assert check_selection_bruteforce(orc.select_layers)


def test_selection_nan_orders_last():
    """A NaN epsilon (a failed solve) orders after every number, NaNs by layer index:
    pinned to NumPy's stable argsort, which sorts NaN to the end in index order."""
    g = np.random.default_rng(41)
    for N in (1, 2, 5, 9, 30):
        for _ in range(20):
            eps = np.round(g.random(N) * 4) / 4
            eps[g.random(N) < 0.3] = np.nan
            order = np.argsort(eps, kind="stable")
            for K in range(N + 1):
                mask, idx = orc.select_layers(eps, K)
                assert idx.tolist() == sorted(order[:K].tolist())
                assert int(mask.sum()) == K and all(mask[idx] == 1)
    # a layer with a NaN epsilon is chosen only once every finite one is
    mask, idx = orc.select_layers([np.nan, 2.0, np.nan, 1.0], 3)
    assert idx.tolist() == [0, 1, 3]


def test_num_selected():
    assert orc.num_selected(0.5, 30) == 15 and orc.num_selected(0.5, 40) == 20
    assert orc.num_selected(0.25, 30) == 7 and orc.num_selected(0.25, 40) == 10
    assert orc.num_selected(0.0, 30) == 0 and orc.num_selected(0.7, 10) == 7
    assert orc.num_selected(0.3, 10) == 3 and orc.num_selected(1.0, 7) == 7


# ---------------------------------------------------------------------------
# P7: KV accounting reproduces the pages' Table 2
# ---------------------------------------------------------------------------
def test_kv_retained_reproduces_table2():
    with open(os.path.join(GOLDEN, "table2_kv_retained.json")) as f:
        rows = json.load(f)["rows"]
    by = {}
    for r in rows:
        by.setdefault(r["backbone"], []).append(r)
    for backbone, rs in by.items():
        # one history fraction h = 1 - 1/n (n an integer frame ratio) must explain every row
        fits = []
        for n in range(2, 40):
            h = 1.0 - 1.0 / n
            if all(abs(100 * orc.kv_retained_fraction(r["x"], h) - r["remaining_pct"]) <= 0.05 + 1e-9 for r in rs):
                fits.append(n)
        assert fits, backbone
    # LongLive's three rows share one history fraction (11/12)
    assert all(abs(100 * orc.kv_retained_fraction(r["x"], 11 / 12) - r["remaining_pct"]) <= 0.05
               for r in by["LongLive"])


# ---------------------------------------------------------------------------
# P8: the split costs the same dot products as full attention
# ---------------------------------------------------------------------------
def test_flop_identity():
    for sh in (si.SHAPE_1P3B, si.SHAPE_14B, si.TINY):
        nl, nh = len(sh.local_rows), len(sh.hist_rows)
        assert nl + nh == sh.Lkv
        f_split = orc.attention_flops(sh.Lq, nl, sh.H, sh.d) + orc.attention_flops(sh.Lq, nh, sh.H, sh.d)
        assert f_split == orc.attention_flops(sh.Lq, sh.Lkv, sh.H, sh.d)
    assert orc.attention_flops(4680, 32760, 12, 128) == pytest.approx(0.942e12, rel=1e-3)


def test_local_projection_definition():
    sh = si.TINY
    d = si.iid_qkv(sh, "f32", ("pin", "proj"))
    W = si.projection_weight(sh.D, sh.D, ("pin", "proj"))
    dW = 0.01 * np.random.default_rng(15).standard_normal((sh.D, sh.D))
    Y = orc.local_projection(sh, d["q"], d["k"], d["v"], W, dW)
    out = orc.split_attention(sh, d["q"], d["k"], d["v"])
    assert np.allclose(Y[0], orc.heads_to_rows(out["O_loc"]) @ (W + dW), atol=1e-13)


@pytest.mark.parametrize("layout", [
    dict(sink_frames=2, hist_begin=2, hist_end=6, cur_begin=6, cur_end=8, kv_frames=9),
    dict(sink_frames=0, hist_begin=0, hist_end=3, cur_begin=3, cur_end=5, kv_frames=5),
    dict(sink_frames=3, hist_begin=0, hist_end=0, cur_begin=2, cur_end=4, kv_frames=4),
    dict(sink_frames=5, hist_begin=0, hist_end=0, cur_begin=1, cur_end=3, kv_frames=6),
])
def test_eviction_keeps_exactly_the_local_frames(layout):
    """Evicting history keeps the sink and current frames, in frame order, and
    drops everything else [DE-summary 2, "Speichereffiziente Inferenz"]: checked
    frame by frame, and local attention over the evicted buffer equals local
    attention over the original (same keys, same order: identical arithmetic)."""
    sh = si.AttnShape(B=2, H=2, d=8, tpf=3, **layout)
    d = si.iid_qkv(sh, "f32", ("pin", "evict"))
    kept_frames = [f for f in range(sh.kv_frames) if f < sh.sink_frames or sh.cur_begin <= f < sh.cur_end]
    for name in ("k", "v"):
        ev = orc.evict_history(sh, d[name])
        brute = np.concatenate([d[name][:, f * sh.tpf:(f + 1) * sh.tpf] for f in kept_frames], axis=1)
        assert np.array_equal(ev, brute)
    es = orc.evicted_shape(sh)
    assert es.kv_frames == len(kept_frames) and es.hist_end == es.hist_begin
    ek, ev_ = orc.evict_history(sh, d["k"]), orc.evict_history(sh, d["v"])
    a = orc.split_attention(sh, d["q"], d["k"], d["v"])
    b = orc.split_attention(es, d["q"], ek, ev_)
    assert np.array_equal(a["O_loc"], b["O_loc"]) and np.array_equal(a["L_loc"], b["L_loc"])
    assert np.all(np.isneginf(b["L_hist"]))


def test_restore_is_the_inverse_of_eviction():
    sh = si.AttnShape(B=2, H=2, d=8, tpf=3, sink_frames=2, hist_begin=2, hist_end=6, cur_begin=6, cur_end=8,
                      kv_frames=9)
    d = si.iid_qkv(sh, "f32", ("pin", "restore"))
    sentinel = np.full_like(d["k"], 7.0)
    back = orc.restore_history(sh, orc.evict_history(sh, d["k"]), sentinel)
    local = np.zeros(sh.kv_frames * sh.tpf, bool)
    for f in list(range(sh.sink_frames)) + list(range(sh.cur_begin, sh.cur_end)):
        local[f * sh.tpf:(f + 1) * sh.tpf] = True
    assert np.array_equal(back[:, local], d["k"][:, local])
    assert np.all(back[:, ~local] == 7.0)


# ---------------------------------------------------------------------------
# mutation tests: plausible mistakes planted in copies of oracle functions
# ---------------------------------------------------------------------------
def test_mutant_plain_average_merge_is_caught():
    def average_merge(oa, la, ob, lb):
        L = np.logaddexp(la, lb)
        return 0.5 * (oa + ob), L
    assert not check_merge_vs_monolithic(average_merge)


def test_mutant_swapped_merge_weights_is_caught():
    def swapped(oa, la, ob, lb):
        L = np.logaddexp(la, lb)
        wa, wb = np.exp(la - L), np.exp(lb - L)
        return wb[..., None] * oa + wa[..., None] * ob, L
    assert not check_merge_vs_monolithic(swapped)


def test_mutant_missing_scale_is_caught():
    def unscaled(q, k, v, scale):
        return orc.attend_group(q, k, v, 1.0)
    assert not check_group_vs_brute(unscaled)


def test_mutant_residual_sign_is_caught():
    def wrong_sign_stats(A_loc, A_full, W):
        G, C, r2 = orc.absorption_stats(A_loc, A_full, W)
        return G, -C, r2
    assert not check_exact_absorption(wrong_sign_stats, orc.ridge_solve, orc.eps_direct)


def test_mutant_transposed_cross_stat_is_caught():
    def transposed(A_loc, A_full, W):
        R = (A_full - A_loc) @ W
        return A_loc.T @ A_loc, (R.T @ A_loc).T[:, ::-1], float(np.sum(R * R))
    assert not check_exact_absorption(transposed, orc.ridge_solve, orc.eps_direct)


def test_mutant_dropped_lambda_is_caught():
    def no_lambda(G, C, lam):
        return orc.ridge_solve(G, C, 0.0)
    assert not check_normal_equations(orc.absorption_stats, no_lambda, lam=0.7)


def test_mutant_largest_eps_selection_is_caught():
    def largest(eps, K):
        return orc.select_layers(-np.asarray(eps), K)
    assert not check_selection_bruteforce(largest)


# ---------------------------------------------------------------------------
# W8A8: the 8-bit formats and the quantised projection
# ---------------------------------------------------------------------------
def e4m3_grid_by_enumeration():
    """Every positive finite e4m3 value, listed from the format's bit fields with Python floats."""
    vals = [m * 2.0 ** -9 for m in range(1, 8)]                      # subnormals
    for e in range(1, 16):
        for m in range(8):
            if e == 15 and m == 7:
                continue                                              # NaN
            vals.append((1 + m / 8) * 2.0 ** (e - 7))
    return sorted(vals)


def test_e4m3_decode_matches_the_format_definition():
    grid = e4m3_grid_by_enumeration()
    assert len(grid) == 126 and grid[-1] == 448.0 and grid[0] == 2.0 ** -9 and grid[7] == 2.0 ** -6
    v = orc.e4m3_decode(np.arange(256, dtype=np.uint8))
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF]) and np.isnan(v).sum() == 2
    assert v[0x00] == 0.0 and v[0x80] == 0.0 and np.signbit(v[0x80])
    pos = v[1:0x7F]
    assert list(pos) == grid                                         # codes 0x01..0x7E in increasing order
    assert np.array_equal(v[0x81:0xFF], -pos)


def test_e4m3_round_is_the_nearest_grid_value_ties_to_even():
    grid = np.array(e4m3_grid_by_enumeration())
    assert np.array_equal(orc.e4m3_round(grid), grid)
    assert np.array_equal(orc.e4m3_round(-grid), -grid)
    full = np.concatenate([[0.0], grid])
    codes = np.arange(0, 127)                                        # code of full[i] is i
    mids = (full[:-1] + full[1:]) / 2
    got = orc.e4m3_round(mids)
    even = np.where(codes[:-1] % 2 == 0, full[:-1], full[1:])        # the neighbour with an even code
    assert np.array_equal(got, even)
    # off-midpoint values go to the nearer neighbour
    lo = full[:-1] + (full[1:] - full[:-1]) * 0.49
    hi = full[:-1] + (full[1:] - full[:-1]) * 0.51
    assert np.array_equal(orc.e4m3_round(lo), full[:-1]) and np.array_equal(orc.e4m3_round(hi), full[1:])
    # saturation
    assert list(orc.e4m3_round(np.array([448.0, 460.0, 464.0, 1e6, -1e30]))) == [448, 448, 448, 448, -448]


def test_e4m3_round_agrees_with_torch_float8_in_range():
    torch = pytest.importorskip("torch")
    x = np.random.default_rng(11).standard_normal(200000) * np.exp(np.random.default_rng(12).uniform(-12, 6, 200000))
    x = x[np.abs(x) <= 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(orc.e4m3_round(x), ref)


def test_int8_rounding_is_half_to_even_and_clamped():
    t = np.array([0.5, 1.5, 2.5, -2.5, -0.5, 2.4999, 126.5, 127.49, 128.0, -300.0, 0.0])
    assert list(orc.q8_round(t, orc.Q8_INT8)) == [0, 2, 2, -2, -0, 2, 126, 127, 127, -127, 0]


@pytest.mark.parametrize("fmt", [orc.Q8_E4M3, orc.Q8_INT8])
def test_quantize_rows_properties(fmt):
    x = si.activation_rows(37, 96, ("pin", "q8", fmt))
    q, s = orc.quantize_rows(x, fmt)
    qmax = orc.Q8_MAX[fmt]
    amax = np.abs(x).max(axis=1)
    assert s.dtype == np.float32 and np.array_equal(s, (amax / np.float32(qmax)).astype(np.float32))
    assert np.all(q[0] == 0) and s[0] == 0                            # zero row
    nz = amax > 0
    # the largest entry of each row lands on +-QMAX exactly
    arg = np.abs(x).argmax(axis=1)
    assert np.all(np.abs(q[np.arange(len(x)), arg])[nz] == qmax)
    assert np.all(np.abs(q) <= qmax)
    # values are on the format's grid
    if fmt == orc.Q8_INT8:
        assert np.array_equal(q, np.round(q))
    else:
        grid = set(e4m3_grid_by_enumeration()) | {0.0}
        assert set(np.abs(q).ravel().tolist()) <= grid
    # dequantisation error: int8 within half a step; e4m3 within half a spacing of the binade
    t = x.astype(np.float64) * (qmax / np.where(nz, amax, 1.0))[:, None]
    if fmt == orc.Q8_INT8:
        assert np.all(np.abs(q - t) <= 0.5 + 1e-5 * qmax)
    else:
        bound = np.maximum(np.abs(t) * 2.0 ** -4, 2.0 ** -10) * (1 + 1e-5)
        assert np.all(np.abs(q - t) <= bound)


def brute_gemm_q8(qa, sa, qw, sw):
    """sum_k qa[m][k] qw[k][n] * sa[m] * sw[n] with exact Python fractions, converted at the end."""
    from fractions import Fraction
    M, K = qa.shape
    N = qw.shape[1]
    y = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            acc = sum(Fraction(float(qa[m, k])) * Fraction(float(qw[k, n])) for k in range(K))
            y[m, n] = float(acc * Fraction(float(sa[m])) * Fraction(float(sw[n])))
    return y


@pytest.mark.parametrize("fmt", [orc.Q8_E4M3, orc.Q8_INT8])
def test_gemm_q8_against_exact_brute_force(fmt):
    x = si.activation_rows(5, 48, ("pin", "gemm", fmt))
    W = si.projection_weight(48, 7, ("pin", "gemm", fmt), "bf16")
    qa, sa = orc.quantize_rows(x, fmt)
    qw, sw = orc.quantize_cols(W, fmt)
    assert qw.shape == (48, 7) and sw.shape == (7,)
    ref = brute_gemm_q8(qa, sa, qw, sw)
    got = np.asarray(orc.gemm_q8(qa, sa, qw, sw, fmt), np.float64)
    if fmt == orc.Q8_INT8:
        # fp32 epilogue: three roundings to nearest fp32
        assert np.all(np.abs(got - ref) <= 3 * 2.0 ** -24 * np.abs(ref) + 1e-45)
    else:
        assert np.allclose(got, ref, rtol=1e-15, atol=0)


@pytest.mark.parametrize("fmt", [orc.Q8_E4M3, orc.Q8_INT8])
def test_w8a8_projection_is_within_the_quantisation_bound(fmt):
    """|A W - deq(A) deq(W)| <= sum_k |a||dW| + |da||W| + |da||dW| with the per-element errors."""
    A = si.activation_rows(40, 256, ("pin", "w8a8", fmt))[2:]
    W = si.projection_weight(256, 24, ("pin", "w8a8", fmt), "bf16")
    qa, sa = orc.quantize_rows(A, fmt)
    qw, sw = orc.quantize_cols(W, fmt)
    Ad = qa * sa[:, None].astype(np.float64)
    Wd = qw * sw[None, :].astype(np.float64)
    dA, dWq = np.abs(A - Ad), np.abs(W - Wd)
    bound = np.abs(A) @ dWq + dA @ np.abs(W) + dA @ dWq
    y = np.asarray(orc.gemm_q8(qa, sa, qw, sw, fmt), np.float64)
    exact = A.astype(np.float64) @ W.astype(np.float64)
    assert np.all(np.abs(y - exact) <= bound * (1 + 1e-5) + 1e-6 * np.abs(exact))
    # and the product stays close: a few percent relative error (the 20x outlier
    # channels of the rows set their scales, which coarsens int8 most)
    rel = np.linalg.norm(y - exact) / np.linalg.norm(exact)
    assert rel < 0.06, rel


def test_mutant_scale_of_the_wrong_side_is_caught():
    x = si.activation_rows(5, 48, ("pin", "gemm", 1))
    W = si.projection_weight(48, 5, ("pin", "gemm", 1), "bf16")
    qa, sa = orc.quantize_rows(x, orc.Q8_INT8)
    qw, sw = orc.quantize_cols(W, orc.Q8_INT8)
    ref = brute_gemm_q8(qa, sa, qw, sw)
    swapped = np.asarray(orc.gemm_q8(qa, sw, qw, sa, orc.Q8_INT8), np.float64)
    assert not np.allclose(swapped, ref, rtol=1e-6)


def test_bf16_round_agrees_with_torch_bfloat16():
    torch = pytest.importorskip("torch")
    g = np.random.default_rng(13)
    x = (g.standard_normal(100000) * np.exp(g.uniform(-30, 30, 100000))).astype(np.float32)
    # exact ties: fp32 values whose low 16 bits are 0x8000, with odd and even kept parts
    ties = ((np.arange(0x3F80, 0x3F80 + 1000, dtype=np.uint32) << 16) | np.uint32(0x8000)).view(np.float32)
    x = np.concatenate([x, ties, -ties])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(orc.bf16_round(x), ref)
    # ties go to the even kept part
    kept = (ties.view(np.uint32) >> 16)
    got = orc.bf16_round(ties).astype(np.float32).view(np.uint32) >> 16
    assert np.all(got % 2 == 0) and np.all((got == kept) | (got == kept + 1))


@pytest.mark.parametrize("fmt", [orc.Q8_E4M3, orc.Q8_INT8])
def test_local_projection_q8_reduces_to_the_unquantised_step(fmt):
    """The W8A8 step approximates A_loc W_new within the quantisation bound of its own operands."""
    sh = si.AttnShape(B=1, H=2, d=16, tpf=3, sink_frames=1, hist_begin=1, hist_end=3, cur_begin=3, cur_end=5,
                      kv_frames=5)
    data = si.iid_qkv(sh, "f32", ("pin", "lq8"))
    W = si.projection_weight(sh.D, 8, ("pin", "lq8"))
    y8 = orc.local_projection_q8(sh, data["q"], data["k"], data["v"], W, fmt)
    y = orc.local_projection(sh, data["q"], data["k"], data["v"], W)
    A = orc.bf16_round(orc.local_projection(sh, data["q"], data["k"], data["v"], np.eye(sh.D)).reshape(-1, sh.D))
    qa, sa = orc.quantize_rows(A, fmt)
    qw, sw = orc.quantize_cols(W, fmt)
    A0 = orc.local_projection(sh, data["q"], data["k"], data["v"], np.eye(sh.D)).reshape(-1, sh.D)
    dA = np.abs(A0 - qa * sa[:, None].astype(np.float64))
    dW = np.abs(W - qw * sw[None, :].astype(np.float64))
    bound = np.abs(A0) @ dW + dA @ np.abs(W) + dA @ dW
    assert np.all(np.abs(y8.reshape(-1, 8) - y.reshape(-1, 8)) <= bound * (1 + 1e-5) + 1e-12)


# ---------------------------------------------------------------------------
# mutation tests of the W8A8 oracle: a planted mistake fails a pin
# ---------------------------------------------------------------------------
def check_e4m3_round(fn) -> bool:
    """The midpoint and saturation pins of test_e4m3_round_is_the_nearest_grid_value_ties_to_even."""
    grid = np.array(e4m3_grid_by_enumeration())
    full = np.concatenate([[0.0], grid])
    mids = (full[:-1] + full[1:]) / 2
    even = np.where(np.arange(126) % 2 == 0, full[:-1], full[1:])
    return (np.array_equal(fn(mids), even) and np.array_equal(fn(grid), grid)
            and fn(np.array([1e6]))[0] == 448.0)


def check_quantize_rows(fn, fmt) -> bool:
    """Per-row scale and the largest entry of each row on +-QMAX."""
    x = si.activation_rows(37, 96, ("pin", "q8", fmt))
    q, s = fn(x, fmt)
    amax = np.abs(x).max(axis=1)
    nz = amax > 0
    arg = np.abs(x).argmax(axis=1)
    return (np.array_equal(s, (amax / np.float32(orc.Q8_MAX[fmt])).astype(np.float32))
            and bool(np.all(np.abs(q[np.arange(len(x)), arg])[nz] == orc.Q8_MAX[fmt])))


def check_gemm_q8(fn) -> bool:
    x = si.activation_rows(5, 48, ("pin", "gemm", 0))
    W = si.projection_weight(48, 7, ("pin", "gemm", 0), "bf16")
    qa, sa = orc.quantize_rows(x, orc.Q8_E4M3)
    qw, sw = orc.quantize_cols(W, orc.Q8_E4M3)
    return np.allclose(np.asarray(fn(qa, sa, qw, sw, orc.Q8_E4M3), np.float64), brute_gemm_q8(qa, sa, qw, sw),
                       rtol=1e-12, atol=0)


def test_w8a8_pins_accept_the_oracle():
    assert check_e4m3_round(orc.e4m3_round)
    assert check_quantize_rows(orc.quantize_rows, orc.Q8_E4M3) and check_quantize_rows(orc.quantize_rows, orc.Q8_INT8)
    assert check_gemm_q8(orc.gemm_q8)


def test_mutant_e4m3_ties_away_from_zero_is_caught():
    def ties_away(x):
        x = np.asarray(x, np.float64)
        a = np.abs(x)
        _, ex = np.frexp(a)
        quantum = np.ldexp(1.0, np.maximum(ex - 1, -6) - 3)
        q = np.minimum(np.floor(a / quantum + 0.5) * quantum, 448.0)
        return np.copysign(q, x)
    assert not check_e4m3_round(ties_away)


def test_mutant_e4m3_without_saturation_is_caught():
    def no_sat(x):
        x = np.asarray(x, np.float64)
        a = np.abs(x)
        _, ex = np.frexp(a)
        quantum = np.ldexp(1.0, np.maximum(ex - 1, -6) - 3)
        return np.copysign(np.rint(a / quantum) * quantum, x)
    assert not check_e4m3_round(no_sat)


def test_mutant_per_tensor_scale_is_caught():
    def per_tensor(x, fmt):
        x32 = np.asarray(x, np.float32)
        amax = np.float32(np.abs(x32).max())
        qmax = np.float32(orc.Q8_MAX[fmt])
        s = np.full(x32.shape[0], amax / qmax, np.float32)
        return orc.q8_round((x32 * (qmax / amax)).astype(np.float64), fmt), s
    assert not check_quantize_rows(per_tensor, orc.Q8_INT8)


def test_mutant_gemm_q8_dropped_column_scale_is_caught():
    def no_sw(qa, sa, qw, sw, fmt):
        return orc.gemm_q8(qa, sa, qw, np.ones_like(sw), fmt)
    assert not check_gemm_q8(no_sw)


# ---------------------------------------------------------------------------
# properties of the 8-bit and bf16 roundings over random inputs (hypothesis)
# ---------------------------------------------------------------------------
from hypothesis import given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402

_finite = st.floats(min_value=-1e4, max_value=1e4, allow_nan=False, allow_infinity=False, width=32)


@settings(max_examples=200, deadline=None)
@given(st.lists(_finite, min_size=2, max_size=64))
def test_e4m3_round_is_monotone_idempotent_and_odd(xs):
    x = np.sort(np.asarray(xs, np.float64))
    q = orc.e4m3_round(x)
    assert np.all(np.diff(q) >= 0)                      # monotone
    assert np.array_equal(orc.e4m3_round(q), q)         # idempotent
    assert np.array_equal(orc.e4m3_round(-x), -q)       # odd
    assert np.all(np.abs(q) <= 448.0)


@settings(max_examples=200, deadline=None)
@given(st.lists(_finite, min_size=2, max_size=64))
def test_bf16_round_is_monotone_and_idempotent(xs):
    x = np.sort(np.asarray(xs, np.float32))
    q = orc.bf16_round(x)
    assert np.all(np.diff(q) >= 0)
    assert np.array_equal(orc.bf16_round(q), q)
    # half a unit in the last place: 2^-8 relative, or half the subnormal spacing 2^-133
    assert np.all(np.abs(q - x) <= 2.0 ** -8 * np.abs(x) + 2.0 ** -134)


@settings(max_examples=60, deadline=None)
@given(st.integers(min_value=0, max_value=2 ** 31 - 1), st.integers(min_value=-20, max_value=20),
       st.sampled_from([orc.Q8_E4M3, orc.Q8_INT8]))
def test_quantize_rows_commutes_with_power_of_two_scaling(seed, k, fmt):
    """x -> x 2^k leaves every code unchanged and scales every row's scale by 2^k exactly
    (amax, QMAX / amax and x * inv all scale exactly while no value leaves fp32's normal range)."""
    x = si.round_to_bf16(np.random.default_rng(seed).standard_normal((6, 40)).astype(np.float32))
    q1, s1 = orc.quantize_rows(x, fmt)
    q2, s2 = orc.quantize_rows((x * np.float32(2.0 ** k)).astype(np.float32), fmt)
    assert np.array_equal(q1, q2)
    assert np.array_equal(s2, (s1 * np.float32(2.0 ** k)).astype(np.float32))


# ---------------------------------------------------------------------------
# FP8 attention (the 8-bit reading of the post-switch attention)
# ---------------------------------------------------------------------------
FP8_LAYOUTS = [
    si.AttnShape(B=1, H=2, d=64, tpf=37, sink_frames=1, hist_begin=1, hist_end=5, cur_begin=5, cur_end=6, kv_frames=6),
    si.AttnShape(B=2, H=1, d=32, tpf=50, sink_frames=2, hist_begin=2, hist_end=2, cur_begin=2, cur_end=4, kv_frames=4),
    si.AttnShape(B=1, H=1, d=32, tpf=200, sink_frames=2, hist_begin=2, hist_end=2, cur_begin=0, cur_end=2, kv_frames=2),
    si.AttnShape(B=1, H=1, d=16, tpf=9, sink_frames=1, hist_begin=1, hist_end=30, cur_begin=30, cur_end=33,
                 kv_frames=33),
]


def _dequantised(data):
    out = {}
    for n in ("q", "k", "v"):
        c, s = orc.quantize_heads(data[n])
        out[n] = c * s.astype(np.float64)[:, None, :, None]
    return out


def check_fp8_online_softmax(fn) -> bool:
    """With the weights kept exact, the blockwise algorithm is softmax attention of
    the dequantised Q, K, V (online softmax is exact whatever the blocks)."""
    ok = True
    for i, sh in enumerate(FP8_LAYOUTS):
        data = si.iid_qkv(sh, "bf16", ("pin", "fp8", i))
        got = fn(sh, data["q"], data["k"], data["v"], quantize_p=False)
        dq = _dequantised(data)
        ref = orc.split_attention(sh, dq["q"], dq["k"], dq["v"])
        for n in ("loc", "hist", "full"):
            ok &= np.allclose(got["O_" + n], ref["O_" + n], rtol=0, atol=1e-12)
            fin = np.isfinite(ref["L_" + n])
            ok &= np.array_equal(fin, np.isfinite(got["L_" + n]))
            ok &= np.allclose(got["L_" + n][fin], ref["L_" + n][fin], rtol=0, atol=1e-12)
    return bool(ok)


def test_fp8_attention_without_weight_rounding_is_softmax_of_the_dequantised_inputs():
    assert check_fp8_online_softmax(orc.split_attention_fp8)


def test_fp8_quantize_heads_is_the_row_quantiser_per_head():
    x = si.round_to_bf16(si.rng("pin", "qh").standard_normal((2, 33, 3, 16)).astype(np.float32) *
                         np.array([1.0, 100.0, 1e-3], np.float32)[None, None, :, None])
    q, s = orc.quantize_heads(x)
    for b in range(2):
        for h in range(3):
            amax = np.float32(np.abs(x[b, :, h]).max())
            assert s[b, h] == np.float32(amax / np.float32(448.0))
            assert np.abs(q[b, :, h]).max() == 448.0
            assert np.array_equal(orc.e4m3_round(q[b, :, h]), q[b, :, h])   # codes on the e4m3 grid


def test_fp8_blocks_cover_each_range_in_aligned_128_key_windows():
    g = np.random.default_rng(5)
    for _ in range(200):
        lo = int(g.integers(0, 3000))
        hi = lo + int(g.integers(1, 1500))
        lo2 = hi + int(g.integers(0, 300))
        hi2 = lo2 + int(g.integers(0, 700))
        ranges = [(lo, hi)] + ([(lo2, hi2)] if hi2 > lo2 else [])
        blocks = orc.fp8_blocks(ranges)
        keys = [k for a, b in blocks for k in range(a, b)]
        assert keys == [k for a, b in ranges for k in range(a, b)]          # every key once, in order
        for a, b in blocks:
            w0 = next(r0 - r0 % 16 + 128 * ((a - (r0 - r0 % 16)) // 128) for r0, r1 in ranges if r0 <= a < r1)
            assert w0 % 16 == 0 and w0 <= a < b <= w0 + 128                # inside one aligned window


def test_fp8_weights_on_the_e4m3_grid_pass_exactly():
    """p = 2^(t - m + 6): the block's maximum enters as 64, and a weight of
    1.125 * 2^-7 relative to it (0.5625 after the offset) is an e4m3 normal and
    enters exactly."""
    v8 = np.array([[1.0, -2.0], [3.0, 0.5]])
    t = np.array([[0.0, math.log2(1.125 * 2.0 ** -7)]])
    o, L = orc.attend_group_fp8(t, v8, [(0, 2)])
    w = np.array([64.0, 0.5625])
    assert np.allclose(o[0], (w @ v8) / w.sum(), rtol=0, atol=1e-15)
    assert abs(L[0] - math.log(1.0 + 1.125 * 2.0 ** -7)) < 1e-15


# Three blocks of one row: the second block's maximum is 2.5 above the first's
# (within TAU = 2.75: the reference stays at 0), the third's is 3.0 above it (the
# reference moves to 3 and the earlier sums scale by 2^-3).  Weights by hand:
# block 1: 2^6 = 64; block 2: 2^8.5 = 362.04 -> e4m3 352 (grid step 32 in
# [256, 512)), 2^5 = 32; block 3: 2^6 = 64.
LAZY_T = np.array([[0.0, 2.5, -1.0, 3.0]])
LAZY_V = np.array([[1.0, 0.0], [0.0, 1.0], [2.0, -1.0], [-1.0, 3.0]])
LAZY_BLOCKS = [(0, 1), (1, 3), (3, 4)]


def _lazy_expected():
    acc = (64.0 * LAZY_V[0] + 352.0 * LAZY_V[1] + 32.0 * LAZY_V[2]) / 8.0 + 64.0 * LAZY_V[3]
    l = (64.0 + 2.0 ** 8.5 + 32.0) / 8.0 + 64.0
    return acc / l


def test_fp8_reference_moves_only_past_the_threshold():
    o, L = orc.attend_group_fp8(LAZY_T, LAZY_V, LAZY_BLOCKS)
    assert np.allclose(o[0], _lazy_expected(), rtol=0, atol=1e-14)
    # L keeps the exact weights: the log-sum-exp of the scores (log2 units)
    assert abs(L[0] - math.log(float(np.sum(np.exp2(LAZY_T[0]))))) < 1e-14
    # the largest weight the threshold admits stays below e4m3's 448
    assert 2.0 ** (orc.FP8_P_OFFSET + orc.FP8_TAU) < 448.0


def test_fp8_tie_allowance_covers_weights_on_a_rounding_boundary():
    """Weights 64 and 42 (42 = halfway between the e4m3 codes 40 and 44, so the tie
    rounds to even: 40): the allowance is the code step 4 times |v| over l = 106;
    weights away from every boundary (the three-block example) have none."""
    v8 = np.array([[1.0, -2.0], [3.0, 0.5]])
    t = np.array([[0.0, math.log2(42.0 / 64.0)]])
    o, _, amb = orc.attend_group_fp8(t, v8, [(0, 2)], tie_rel=2.0 ** -14)
    assert np.allclose(o[0], (64.0 * v8[0] + 40.0 * v8[1]) / 106.0, rtol=0, atol=1e-14)
    assert np.allclose(amb[0], 4.0 * np.abs(v8[1]) / 106.0, rtol=0, atol=1e-14)
    # the other rounding of the tie lies at the edge of the allowance
    assert np.allclose(np.abs((64.0 * v8[0] + 44.0 * v8[1]) / 106.0 - o[0]), amb[0], rtol=0, atol=1e-14)
    _, _, amb = orc.attend_group_fp8(LAZY_T, LAZY_V, LAZY_BLOCKS, tie_rel=2.0 ** -14)
    assert np.all(amb == 0)
    # a block maximum within tie_rel of the threshold leaves the reference undecided
    t = np.array([[0.0, 2.75], [0.0, 2.0]])
    _, _, amb = orc.attend_group_fp8(t, v8, [(0, 1), (1, 2)], tie_rel=2.0 ** -14)
    assert np.all(np.isinf(amb[0])) and np.all(np.isfinite(amb[1]))


def test_fp8_tie_allowance_bounds_every_rounding_of_perturbed_weights():
    """Scores moved by a relative 2^-16 give, through the oracle itself, outputs
    that stay within the allowance computed at tie_rel = 2^-14 (brute force over
    seeded perturbations of a small layout)."""
    sh = FP8_LAYOUTS[0]
    data = si.iid_qkv(sh, "bf16", ("pin", "fp8tie"))
    q8, sq = orc.quantize_heads(data["q"])
    k8, sk = orc.quantize_heads(data["k"])
    v8, _ = orc.quantize_heads(data["v"])
    blk = orc.fp8_blocks(orc._runs(orc._hist_rows(sh)))
    g = np.random.default_rng(11)
    for h in range(sh.H):
        c = float(sq[0, h]) * float(sk[0, h]) / math.sqrt(sh.d) / math.log(2.0)
        t = (q8[0, :, h, :] @ k8[0, :, h, :].T) * c
        o, _, amb = orc.attend_group_fp8(t, v8[0, :, h, :], blk, tie_rel=2.0 ** -14)
        for _ in range(5):
            tp = t + np.log2(1.0 + g.uniform(-2.0 ** -16, 2.0 ** -16, t.shape))
            op, _ = orc.attend_group_fp8(tp, v8[0, :, h, :], blk)
            # the exact weights move by 2^-16 too: their own share of the difference
            assert np.all(np.abs(op - o) <= amb + 2.0 ** -15 * np.abs(o) + 1e-12)


def test_mutant_fp8_reference_following_every_maximum_is_caught():
    """A reference that follows the running maximum at every block rounds the
    second block's weights at another place of the grid (64 and 2^2.5 -> 5.5)."""
    def every_block(t, v8, blocks):
        n, d = t.shape[0], v8.shape[1]
        m, l, acc = np.full(n, -np.inf), np.zeros(n), np.zeros((n, d))
        for lo, hi in blocks:
            tb = t[:, lo:hi]
            m_new = np.maximum(m, tb.max(axis=1))
            f = np.where(np.isneginf(m), 0.0, np.exp2(m - m_new))
            acc, l, m = acc * f[:, None], l * f, m_new
            p = np.exp2(tb - m[:, None] + orc.FP8_P_OFFSET)
            l += p.sum(axis=1)
            acc += orc.e4m3_round(p) @ v8[lo:hi]
        return acc / l[:, None]
    assert not np.allclose(every_block(LAZY_T, LAZY_V, LAZY_BLOCKS)[0], _lazy_expected(), rtol=0, atol=1e-6)


def test_fp8_weight_rounding_stays_within_its_bound():
    """With e4m3 weights the output moves by at most 2^-4 of sum_j w_j |v_j| (normal
    weights) plus 2^-10 per subnormal weight over l >= 2^6 (the key that set the
    reference weighs 2^6); L is unchanged (the
    normaliser keeps the exact weights); and the rounding is really applied."""
    for i, sh in enumerate(FP8_LAYOUTS):
        data = si.iid_qkv(sh, "bf16", ("pin", "fp8b", i))
        got = orc.split_attention_fp8(sh, data["q"], data["k"], data["v"])
        exact = orc.split_attention_fp8(sh, data["q"], data["k"], data["v"], quantize_p=False)
        dq = _dequantised(data)
        moved = 0.0
        for name, rows in (("loc", orc._local_rows(sh)), ("hist", orc._hist_rows(sh))):
            if len(rows) == 0:
                continue
            for b in range(sh.B):
                for h in range(sh.H):
                    s = (dq["q"][b, :, h] @ dq["k"][b, rows, h].T) / math.sqrt(sh.d)
                    w = np.exp(s - s.max(axis=1, keepdims=True))
                    w /= w.sum(axis=1, keepdims=True)
                    av = np.abs(dq["v"][b, rows, h])
                    bound = 2.0 ** -4 * (w @ av) + 2.0 ** -16 * av.sum(axis=0)[None, :] + 1e-12
                    err = np.abs(got["O_" + name][b, :, h] - exact["O_" + name][b, :, h])
                    assert np.all(err <= bound), (i, name, float((err - bound).max()))
                    moved = max(moved, float(err.max()))
            fin = np.isfinite(exact["L_" + name])
            assert np.allclose(got["L_" + name][fin], exact["L_" + name][fin], rtol=0, atol=1e-12)
        assert moved > 1e-6


def test_mutant_fp8_without_the_weight_offset_is_caught():
    def no_offset(t, v8, blocks, quantize_p=True):
        n, d = t.shape[0], v8.shape[1]
        m, l, acc = np.full(n, -np.inf), np.zeros(n), np.zeros((n, d))
        for lo, hi in blocks:
            tb = t[:, lo:hi]
            m_new = np.maximum(m, tb.max(axis=1))
            f = np.where(np.isneginf(m), 0.0, np.exp2(m - m_new))
            acc, l, m = acc * f[:, None], l * f, m_new
            p = np.exp2(tb - m[:, None])
            l += p.sum(axis=1)
            acc += orc.e4m3_round(p) @ v8[lo:hi]
        return acc / l[:, None], (m + np.log2(l)) * math.log(2.0)
    v8 = np.array([[1.0, -2.0], [3.0, 0.5]])
    t = np.array([[0.0, math.log2(1.125 * 2.0 ** -7)]])
    o, _ = no_offset(t, v8, [(0, 2)])
    w = np.array([64.0, 0.5625])
    assert not np.allclose(o[0], (w @ v8) / w.sum(), rtol=0, atol=1e-15)


def test_mutant_fp8_v_dequantised_with_the_k_scale_is_caught():
    def wrong_v_scale(shape, q, k, v, scale=None, rows=None, quantize_p=True):
        out = orc.split_attention_fp8(shape, q, k, v, scale, rows, quantize_p)
        _, sk = orc.quantize_heads(k)
        _, sv = orc.quantize_heads(v)
        f = (sk.astype(np.float64) / sv.astype(np.float64))[:, None, :, None]
        for n in ("loc", "hist", "full"):
            out["O_" + n] = out["O_" + n] * f
        return out
    assert not check_fp8_online_softmax(wrong_v_scale)
