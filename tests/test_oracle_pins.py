"""Pins of the CPU oracle against what the source pages and mathematics fix.

Each test checks the oracle against something other than itself: a worked
example printed on the pages (tests/golden), a closed form, an invariant, a
special case that reduces to a textbook routine, or brute force on tiny inputs.
The cases are chosen so that a plausible slip in the oracle (an off-by-one
rank, a non-strict mask, a flipped rank direction, a dropped term, a
transposed weight) makes at least one of them fail; tests/test_oracle_mutants.py
plants such slips and checks that.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle as O


def _rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- mask / compaction

def test_teal_worked_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "teal_worked_example.json")))
    x = np.array(g["x"])
    m = O.magnitude_mask(x, g["threshold"])
    assert m.astype(int).tolist() == g["mask"]
    idx, cnt = O.compact(m)
    assert idx.tolist() == g["active_idx"] and cnt == 2
    # y = sparse_x @ W on the printed sparse_x, summed row by row in Python
    W = _rng(0).standard_normal((5, 7))
    y_loop = [sum(g["sparse_x"][i] * W[i, n] for i in range(5)) for n in range(7)]
    y = O.masked_gemv(x, m, W)[0]
    np.testing.assert_allclose(y, y_loop, rtol=0, atol=1e-14)


def test_mask_is_strict_at_threshold():
    # values equal to t are zeroed: |x| > t, not >=
    x = np.array([0.5, -0.5, 0.50001, 0.0])
    assert O.magnitude_mask(x, 0.5).tolist() == [False, False, True, False]


def test_compact_ascending_and_union():
    m = np.array([[1, 0, 0, 1, 0, 1], [0, 0, 1, 1, 0, 0]], dtype=bool)
    assert O.compact(m[0])[0].tolist() == [0, 3, 5]
    assert O.union_mask(m).astype(int).tolist() == [1, 0, 1, 1, 0, 1]


# ---------------------------------------------------------------- calibration

@pytest.mark.parametrize("p", [0.25, 0.4, 0.5, 0.65, 0.9, 0.1, 0.7, 1.0])
def test_calibration_order_statistic_invariant(p):
    # bf16-like data with many ties: t is the r-th smallest iff
    # #{a < t} < r <= #{a <= t} and t is a data value.
    a = np.round(np.abs(_rng(1).laplace(size=(64, 33))) * 8) / 8
    N = a.size
    t = O.calibrate_threshold(a, p)
    r = math.ceil(round(p * N, 9))
    assert (a < t).sum() < r <= (a <= t).sum()
    assert t in set(a.ravel().tolist())


@pytest.mark.parametrize("p", [0.25, 0.4, 0.5, 0.65, 0.9])
def test_calibration_hits_target_fraction(p):
    # [TEAL] slide 8: t_p zeroes the target fraction of calibration magnitudes.
    # Brute force over candidate thresholds: t is the smallest data value whose
    # strict mask zeroes at least p of the pooled draws.
    a = np.abs(np.round(_rng(2).laplace(size=(16, 40)) * 4) / 4)
    flat = a.ravel()
    t = O.calibrate_threshold(a, p)
    zero_frac = lambda c: np.mean(~O.magnitude_mask(flat, c))
    assert zero_frac(t) >= p - 1e-12
    cands = sorted(set(flat.tolist()))
    best = min(c for c in cands if np.mean(flat <= c) >= p - 1e-12)
    assert t == best
    # with distinct continuous values the zeroed fraction is exactly ceil(pN)/N
    # (N = 1001 makes p*N fractional, so ceil and floor differ)
    c = np.abs(_rng(3).laplace(size=1001))
    tc = O.calibrate_threshold(c, p)
    assert np.sum(~O.magnitude_mask(c, tc)) == math.ceil(round(p * 1001, 9))


def test_calibration_rank_decimal_products():
    assert O.calibration_rank(0.7, 100) == 70
    assert O.calibration_rank(0.65, 16384) == 10650
    assert O.calibration_rank(0.5, 16384) == 8192
    assert O.calibration_rank(0.1, 10) == 1
    assert O.calibrate_threshold(np.arange(1.0, 11.0), 0.7) == 7.0


def test_sparsity_zero_is_dense_gemv():
    # [TEAL] slide 15 baseline: sparsity 0 is the dense product.
    calib = _rng(4).laplace(size=(8, 12))
    t = O.calibrate_threshold(calib, 0.0)
    assert t == -math.inf
    x = _rng(5).laplace(size=(2, 12))
    W = _rng(6).standard_normal((12, 9))
    m = O.magnitude_mask(x, t)
    assert m.all()
    dense = [[sum(x[b, i] * W[i, n] for i in range(12)) for n in range(9)] for b in range(2)]
    np.testing.assert_allclose(O.masked_gemv(x, m, W), dense, rtol=0, atol=1e-13)


def test_sparsity_one_is_zero_output():
    calib = np.abs(_rng(7).laplace(size=(8, 12)))
    t = O.calibrate_threshold(calib, 1.0)
    assert t == calib.max()
    m = O.magnitude_mask(calib, t)
    assert not m.any() and O.compact(m[0])[1] == 0
    W = _rng(8).standard_normal((12, 4))
    assert np.all(O.masked_gemv(calib, m, W) == 0.0)


# ---------------------------------------------------------------- masked product

def test_masked_gemv_all_masks_brute_force():
    K, N = 10, 6
    x = _rng(9).laplace(size=K)
    W = _rng(10).standard_normal((K, N))
    for bits in range(1 << K):
        m = np.array([(bits >> i) & 1 for i in range(K)], dtype=bool)
        want = np.zeros(N)
        for i in range(K):
            if m[i]:
                want += x[i] * W[i]
        np.testing.assert_allclose(O.masked_gemv(x, m, W)[0], want, rtol=0, atol=1e-12)


def test_masked_gemv_linearity_and_orientation():
    K, N = 12, 5  # K != N so a transposed W cannot pass
    x = _rng(11).laplace(size=K)
    W = _rng(12).standard_normal((K, N))
    m1 = np.zeros(K, bool); m1[[0, 3, 7]] = True
    m2 = np.zeros(K, bool); m2[[1, 4, 11]] = True
    y = lambda m: O.masked_gemv(x, m, W)[0]
    np.testing.assert_allclose(y(m1 | m2), y(m1) + y(m2), atol=1e-13)
    e = np.zeros(K, bool); e[4] = True
    np.testing.assert_allclose(y(e), x[4] * W[4], atol=0)
    assert O.masked_gemv(x, m1, W).shape == (1, N)


def test_batch_union_equals_batch_one():
    B, K, N = 4, 40, 16
    x = _rng(13).laplace(size=(B, K))
    W = _rng(14).standard_normal((K, N))
    t = 0.9
    m = O.magnitude_mask(x, t)
    yb = O.masked_gemv(x, m, W)
    for b in range(B):
        np.testing.assert_allclose(yb[b], O.masked_gemv(x[b], m[b], W)[0], atol=1e-13)
    # reading only the union rows gives the same result
    u = O.union_mask(m)
    yu = (x[:, u] * m[:, u]) @ W[u]
    np.testing.assert_allclose(yb, yu, atol=1e-13)


# ---------------------------------------------------------------- top-k / scores

def test_topk_brute_force_with_ties():
    n = 10
    rng = _rng(15)
    for trial in range(40):
        s = rng.integers(0, 4, size=n).astype(float)  # many ties
        for k in range(0, n + 1):
            m = O.topk_mask(s, k)
            best = None
            for comb in itertools.combinations(range(n), k):
                tot = s[list(comb)].sum()
                if best is None or tot > best[0]:
                    best = (tot, comb)  # combinations() is lexicographic
            assert tuple(np.flatnonzero(m)) == best[1], (s, k)


def test_keep_counts_for_phi2_ffn():
    assert [O.keep_count(f, 10240) for f in (0.3, 0.5, 0.7)] == [3072, 5120, 7168]


def test_gxo_score_is_rounded_fp32_product():
    g = np.array([1.5, -2.0, 3.0], dtype=np.float32)
    h = np.array([2.0, 0.25, -0.5], dtype=np.float32)
    assert O.gxo_score(g, h).tolist() == [3.0, 0.5, 1.5]
    assert O.gxo_score(g, h).dtype == np.float32
    # one rounding: (1 + 2^-12)^2 = 1 + 2^-11 + 2^-24 -> rounds to even 1 + 2^-11
    a = np.array([1 + 2.0 ** -12], dtype=np.float32)
    assert O.gxo_score(a, a)[0] == np.float32(1 + 2.0 ** -11)


def test_corrected_gxo_closed_form():
    g = np.array([3.0, 4.0])
    h = np.array([1.0, -2.0])
    # ||g|| = 5: s = g*h + 0.5*|h|*5
    assert O.corrected_gxo_score(g, h).tolist() == [3.0 + 2.5, -8.0 + 5.0]


def test_corrected_gxo_f32_closed_form():
    # ||g||_2 = 5 over both neurons: s = g h + |h| * 5 / 2, all exact in float32
    g = np.array([3.0, 4.0], dtype=np.float32)
    h = np.array([1.0, -2.0], dtype=np.float32)
    s = O.corrected_gxo_score_f32(g, h)
    assert s.dtype == np.float32
    assert s.tolist() == [5.5, -3.0]


def test_corrected_gxo_f32_norm_covers_every_neuron():
    # the norm is the layer's (ATTR "correction term": sum over k = 1..N1),
    # including a neuron whose own output is 0
    g = np.array([0.0, 0.0, 12.0], dtype=np.float32)
    h = np.array([1.0, -1.0, 0.0], dtype=np.float32)
    assert O.corrected_gxo_score_f32(g, h).tolist() == [6.0, 6.0, 0.0]


def test_corrected_gxo_f32_keeps_the_sign():
    # GxO -4 vs 0.5: |GxO| ranks neuron 0 first; the corrected signed score
    # -4 + 4 sqrt(2) / 2 = -1.17 < 0.5 + 0.5 sqrt(2) / 2 = 0.85 ranks neuron 1 first
    g = np.array([1.0, 1.0], dtype=np.float32)
    h = np.array([-4.0, 0.5], dtype=np.float32)
    s = O.corrected_gxo_score_f32(g, h)
    assert s[0] < 0 < s[1]
    assert O.topk_mask(s, 1).tolist() == [False, True]
    assert O.topk_mask(O.gxo_score(g, h), 1).tolist() == [True, False]


def test_corrected_gxo_f32_within_rounding_of_the_fp64_definition():
    rng = np.random.default_rng(11)
    g = rng.standard_normal(4096).astype(np.float32)
    h = rng.standard_normal(4096).astype(np.float32)
    s32 = O.corrected_gxo_score_f32(g, h).astype(np.float64)
    s64 = O.corrected_gxo_score(g, h)
    n = math.sqrt(float(np.sum(g.astype(np.float64) ** 2)))
    scale = np.abs(g.astype(np.float64) * h) + 0.5 * np.abs(h.astype(np.float64)) * n
    assert np.all(np.abs(s32 - s64) <= 4 * 2.0 ** -24 * scale)


def test_static_mask_ffn_limits_and_one_neuron():
    rng = np.random.default_rng(21)
    d, f = 6, 5
    x = rng.standard_normal((2, d))
    Wa, Wb, Wd = rng.standard_normal((d, f)), rng.standard_normal((d, f)), rng.standard_normal((f, d))
    # all kept: the dense GeLU FFN; none kept: zero
    y_all, h = O.ffn_static_mask(x, Wa, Wd, np.ones(f, bool))
    phi = np.array([[0.5 * (1 + math.erf(v / math.sqrt(2))) for v in r] for r in x @ Wa])
    assert np.allclose(y_all, ((x @ Wa) * phi) @ Wd, rtol=1e-12, atol=1e-12)
    assert np.all(O.ffn_static_mask(x, Wa, Wd, np.zeros(f, bool))[0] == 0.0)
    # one kept neuron j: y = h_j * W_d[j, :], with SwiGLU h_j = SiLU(x.Wa_j) (x.Wb_j)
    j = 3
    keep = np.zeros(f, bool)
    keep[j] = True
    y1, _ = O.ffn_static_mask(x, Wa, Wd, keep, act="swiglu", W_b=Wb)
    a, u = x @ Wa[:, j], x @ Wb[:, j]
    hj = a / (1 + np.exp(-a)) * u
    assert np.allclose(y1, hj[:, None] * Wd[j][None, :], rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- GLASS

def test_glass_ranks_direction():
    s = np.array([0.1, 0.9, 0.5, 0.9])
    # most important gets n; equal scores: lower index is more important
    assert O.glass_ranks(s).tolist() == [1, 4, 2, 3]


@pytest.mark.parametrize("lam,which", [(0.0, "local"), (1.0, "global")])
def test_glass_lambda_endpoints_reduce_to_single_topk(lam, which):
    rng = _rng(16)
    for _ in range(20):
        sl, sg = rng.random(30), rng.random(30)
        k = int(rng.integers(1, 30))
        want = O.topk_mask(sl if which == "local" else sg, k)
        assert np.array_equal(O.glass_mask(sl, sg, lam, k), want)


@pytest.mark.parametrize("lam", [0.5, 0.3, 0.8])
def test_glass_is_squared_spearman_map(lam):
    # [GLASS] 2.2: the fused order is the MAP consensus ranking under a
    # Mallows-type model with squared Spearman distance: over all rank
    # assignments pi (a permutation of 1..n), the ordering by F minimises
    # (1-lam) sum (pi - R_l)^2 + lam sum (pi - R_g)^2.
    rng = _rng(17)
    n = 6
    for _ in range(15):
        Rl = O.glass_ranks(rng.random(n))
        Rg = O.glass_ranks(rng.random(n))
        cost = lambda pi: (1 - lam) * np.sum((pi - Rl) ** 2) + lam * np.sum((pi - Rg) ** 2)
        best = min(cost(np.array(p)) for p in itertools.permutations(range(1, n + 1)))
        F = O.glass_fuse(Rl, Rg, lam)
        pi_F = O.glass_ranks(F)
        assert abs(cost(pi_F) - best) < 1e-9
        # and the kept set is the top-k of that ranking
        for k in range(n + 1):
            assert np.array_equal(O.topk_mask(F, k), pi_F > n - k)


# ---------------------------------------------------------------- activations / FFN

def test_activation_closed_forms(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "activation_closed_forms.json")))
    for v, want in g["silu"].items():
        assert abs(float(O.silu(float(v))) - want) < 1e-15
    for v, want in g["gelu"].items():
        assert abs(float(O.gelu_erf(float(v))) - want) < 1e-15
    assert abs(float(O.gelu_tanh(1.0)) - g["gelu_tanh"]["1.0"]) < 1e-15


def test_ffn_swiglu_identity_weights(golden_dir):
    # With W_g = W_u = W_d = I: g = u = x m_x, h = SiLU(x) x on kept inputs,
    # y = h m_h. Checked against the textbook SiLU values.
    c = json.load(open(os.path.join(golden_dir, "activation_closed_forms.json")))["silu"]
    x = np.array([[1.0, -1.0, 2.0, 0.25]])
    I = np.eye(4)
    y, h, m_x, m_h = O.ffn_swiglu(x, 0.5, I, I, I, 0.5)
    assert m_x.tolist() == [[True, True, True, False]]
    want_h = [c["1.0"] * 1.0, c["-1.0"] * -1.0, c["2.0"] * 2.0, 0.0]
    np.testing.assert_allclose(h[0], want_h, atol=1e-15)
    want_y = [v if abs(v) > 0.5 else 0.0 for v in want_h]
    np.testing.assert_allclose(y[0], want_y, atol=1e-15)
    # gate and up are not interchangeable: SiLU is applied to the gate only
    Wg = np.diag([1.0, 1.0, 1.0, 1.0]); Wu = np.diag([2.0, 2.0, 2.0, 2.0])
    _, h2, _, _ = O.ffn_swiglu(x, 0.5, Wg, Wu, I, -math.inf)
    np.testing.assert_allclose(h2[0, :3], [2 * c["1.0"], -2 * c["-1.0"], 4 * c["2.0"]], atol=1e-15)


def test_ffn_dense_limits_equal_loops():
    d, f = 5, 7
    rng = _rng(18)
    x = rng.laplace(size=(1, d))
    Wg, Wu, Wd = rng.standard_normal((d, f)), rng.standard_normal((d, f)), rng.standard_normal((f, d))
    y, h, _, _ = O.ffn_swiglu(x, -math.inf, Wg, Wu, Wd, -math.inf)
    for j in range(f):
        gj = sum(x[0, i] * Wg[i, j] for i in range(d))
        uj = sum(x[0, i] * Wu[i, j] for i in range(d))
        assert abs(h[0, j] - gj / (1 + math.exp(-gj)) * uj) < 1e-12
    for n in range(d):
        assert abs(y[0, n] - sum(h[0, j] * Wd[j, n] for j in range(f))) < 1e-12
    # a down threshold above every |h| gives y = 0
    y0, _, _, m_h = O.ffn_swiglu(x, -math.inf, Wg, Wu, Wd, float(np.abs(h).max()))
    assert not m_h.any() and np.all(y0 == 0)


def test_gelu_topk_down_keeps_topk_rows():
    n, d = 12, 4
    rng = _rng(19)
    h = rng.standard_normal(n).astype(np.float32)
    g = rng.standard_normal(n).astype(np.float32)
    W2 = rng.standard_normal((n, d))
    y, m = O.ffn_gelu_topk_down(h, g, W2, 5)
    s = [abs(float(np.float32(g[i]) * np.float32(h[i]))) for i in range(n)]
    keep = sorted(range(n), key=lambda i: (-s[i], i))[:5]
    assert sorted(np.flatnonzero(m).tolist()) == sorted(keep)
    np.testing.assert_allclose(y, sum(float(h[i]) * W2[i] for i in keep), atol=1e-12)


# ---------------------------------------------------------------- MoE

def test_moe_route_brute_force():
    rng = _rng(20)
    for _ in range(20):
        z = np.round(rng.standard_normal(10), 1)  # ties happen
        ex, w = O.moe_route(z, 3)
        assert abs(w.sum() - 1.0) < 1e-15
        best = None
        for comb in itertools.combinations(range(10), 3):
            tot = sum(math.exp(z[i]) for i in comb)
            if best is None or tot > best[0] + 1e-15:
                best = (tot, comb)
        assert tuple(sorted(ex.tolist())) == best[1]
        p = np.exp(z) / np.exp(z).sum()
        np.testing.assert_allclose(w, p[ex] / p[ex].sum(), rtol=1e-14)
        _, w_raw = O.moe_route(z, 3, renormalize=False)
        np.testing.assert_allclose(w_raw, p[ex], rtol=1e-14)


def test_moe_zero_sparsity_is_dense_swiglu_expert():
    d, f = 6, 5
    rng = _rng(21)
    x = rng.laplace(size=d)
    Wg, WuT, Wd = rng.standard_normal((d, f)), rng.standard_normal((f, d)), rng.standard_normal((f, d))
    y, a, m = O.moe_expert(x, Wg, WuT, Wd, -math.inf)
    assert m.all()
    y_ffn, _, _, _ = O.ffn_swiglu(x[None], -math.inf, Wg, WuT.T, Wd, -math.inf)
    np.testing.assert_allclose(y, y_ffn[0], atol=1e-12)
    # mask selects exactly the neurons with |SiLU(gate)| above t_e
    t = float(np.median(np.abs(a)))
    y2, _, m2 = O.moe_expert(x, Wg, WuT, Wd, t)
    assert m2.tolist() == (np.abs(a) > t).tolist()
    u = WuT @ x
    np.testing.assert_allclose(y2, sum(a[j] * u[j] * Wd[j] for j in range(f) if m2[j]), atol=1e-12)


def test_moe_layer_combines_experts_and_shared():
    E, d, f, fs, k = 5, 4, 3, 6, 2
    rng = _rng(22)
    x = rng.laplace(size=(2, d))
    logits = rng.standard_normal((2, E))
    Wg, WuT, Wd = rng.standard_normal((E, d, f)), rng.standard_normal((E, f, d)), rng.standard_normal((E, f, d))
    te = np.full(E, 0.1)
    Sg, Su, Sd = rng.standard_normal((d, fs)), rng.standard_normal((d, fs)), rng.standard_normal((fs, d))
    y = O.moe_layer(x, logits, Wg, WuT, Wd, te, k, Sg, Su, Sd)
    for t in range(2):
        p = np.exp(logits[t]) / np.exp(logits[t]).sum()
        sel = np.argsort(-p)[:k]
        want = sum(p[e] / p[sel].sum() * O.moe_expert(x[t], Wg[e], WuT[e], Wd[e], te[e])[0] for e in sel)
        want = want + O.ffn_swiglu(x[t:t + 1], -math.inf, Sg, Su, Sd, -math.inf)[0][0]
        np.testing.assert_allclose(y[t], want, atol=1e-12)


# ---------------------------------------------------------------- rounding helper

def test_round_to_bf16_and_f16():
    v = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9, 1.0 + 2 ** -9, 65504.0, 1.0 + 2 ** -11])
    bf = O.round_to(v, "bf16")
    assert bf[0] == 1.0          # tie -> even
    assert bf[1] == 1.0 + 2 ** -7
    assert bf[2] == 1.0
    h = O.round_to(v, "f16")
    assert h[3] == 65504.0 and h[4] == 1.0   # tie -> even


# ---------------------------------------------------------------- greedy block allocation

def test_block_error_closed_form_diagonal_weights():
    # W = diag(d): block output y = x * d, so the error at level p is the l2 norm
    # of the dropped activations scaled by d: sqrt(sum over |x| <= t_p of (x d)^2)
    X = _rng(20).laplace(size=(8, 24))
    d = _rng(21).uniform(0.5, 2.0, size=24)
    levels = [0.0, 0.25, 0.5, 0.75, 1.0]
    err, thr = O.block_error_curve(X, np.diag(d), levels)
    for p, e, t in zip(levels, err, thr):
        dropped = np.abs(X) <= t
        assert e == pytest.approx(math.sqrt(((X * d) ** 2)[dropped].sum()), rel=1e-12, abs=1e-15)
    assert err[0] == 0.0                      # dense: no error
    assert err[-1] == pytest.approx(np.linalg.norm(X * d), rel=1e-12)  # all dropped


def test_block_error_uses_the_full_output_change():
    # rectangular W: the error is ||(X m) W - X W||, i.e. the norm of the
    # dropped part pushed through W, row by row in Python
    X = _rng(22).laplace(size=(3, 6))
    W = _rng(23).standard_normal((6, 4))
    err, thr = O.block_error_curve(X, W, [0.5])
    tot = 0.0
    for s in range(3):
        for n in range(4):
            v = sum(X[s, i] * W[i, n] for i in range(6) if abs(X[s, i]) <= thr[0])
            tot += v * v
    assert err[0] == pytest.approx(math.sqrt(tot), rel=1e-12)


def _convex_curves(rng, M, P):
    inc = np.sort(rng.uniform(0.1, 3.0, size=(M, P - 1)), axis=1)  # growing increments
    return np.concatenate([np.zeros((M, 1)), np.cumsum(inc, axis=1)], axis=1)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_greedy_is_optimal_on_convex_curves_brute_force(seed):
    # With equal weights and error curves whose increments grow, raising the
    # block with the smallest growth one level at a time gives the least total
    # error among all allocations with the same number of levels (the classic
    # marginal-allocation result); brute force over every allocation of 3 blocks.
    M, P, step = 3, 5, 0.25
    err = _convex_curves(_rng(100 + seed), M, P)
    for T in range(0, M * (P - 1) + 1):
        lvl = O.greedy_allocate(err, np.ones(M), step, T * step / M)
        assert lvl.sum() == T
        best = min(sum(err[i, a[i]] for i in range(M))
                   for a in itertools.product(range(P), repeat=M) if sum(a) == T)
        assert sum(err[i, lvl[i]] for i in range(M)) == pytest.approx(best, rel=1e-12)


def test_greedy_weighted_overall_sparsity_and_stop():
    # weights 1 and 3: one level (0.5) of block 1 already gives overall 0.375,
    # which is below 0.4; the next level of the cheaper block reaches it
    err = np.array([[0.0, 1.0, 5.0], [0.0, 0.5, 4.0]])
    lvl = O.greedy_allocate(err, [1.0, 3.0], 0.5, 0.4)
    assert lvl.tolist() == [1, 1]
    assert O.overall_sparsity(lvl * 0.5, [1.0, 3.0]) == pytest.approx(0.5)
    assert O.overall_sparsity([0.5, 0.0], [1.0, 3.0]) == pytest.approx(0.125)
    # target 0: every block stays dense; unreachable target: every block ends at its top level
    assert O.greedy_allocate(err, [1.0, 3.0], 0.5, 0.0).tolist() == [0, 0]
    assert O.greedy_allocate(err, [1.0, 3.0], 0.5, 2.0).tolist() == [2, 2]


def test_greedy_compares_growth_per_unit_of_overall_sparsity():
    # block 1 weighs 4x block 0: one level of block 1 gains 4x the overall
    # sparsity, so its growth of 2 counts as 0.5 per unit against block 0's 1;
    # going up on block 1 reaches the 40 % target with half the error of the
    # allocation that raw growths would pick ([2, 1], error 4)
    err = np.array([[0.0, 1.0, 2.0], [0.0, 2.0, 4.0]])
    lvl = O.greedy_allocate(err, [1.0, 4.0], 0.5, 0.4)
    assert lvl.tolist() == [0, 1]
    assert err[0, lvl[0]] + err[1, lvl[1]] == 2.0


def test_greedy_free_block_first_and_ties_to_lower_index():
    # a block that loses nothing is sparsified first; equal growths go to the
    # lower block index
    err = np.array([[0.0, 1.0, 2.0], [0.0, 0.0, 0.0], [0.0, 1.0, 2.0]])
    assert O.greedy_allocate(err, np.ones(3), 0.5, 1 / 3).tolist() == [0, 2, 0]
    assert O.greedy_allocate(err, np.ones(3), 0.5, 0.5).tolist() == [1, 2, 0]
