"""Plausible slips planted in the CPU oracle, to show the pin suite catches them.

Used only by tests/test_oracle_mutants.py, which runs tests/test_oracle_pins.py
in a subprocess with SFX_ORACLE_MUTANT=<name>; tests/conftest.py then swaps the
named oracle function for the mutant below before the pins run. Nothing here
touches a GPU.
"""
import math

import numpy as np


def _mutants(O):
    M = {}

    def calib_off_by_one(calib_abs, p):
        a = np.sort(np.abs(np.asarray(calib_abs, np.float64)).ravel())
        if p <= 0:
            return -math.inf
        r = O.calibration_rank(p, a.size)
        return float(a[min(r, a.size - 1)])
    M["calib_off_by_one"] = ("calibrate_threshold", calib_off_by_one)

    def calib_floor(calib_abs, p):
        a = np.sort(np.abs(np.asarray(calib_abs, np.float64)).ravel())
        if p <= 0:
            return -math.inf
        r = max(1, int(math.floor(p * a.size)))
        return float(a[r - 1])
    M["calib_floor"] = ("calibrate_threshold", calib_floor)

    M["mask_non_strict"] = ("magnitude_mask",
                            lambda x, t: np.abs(np.asarray(x, np.float64)) >= t)

    def topk_ties_high(score, k):
        s = np.asarray(score, np.float64)
        n = s.size
        order = np.lexsort((-np.arange(n), -s))
        m = np.zeros(n, bool)
        m[order[:max(0, min(k, n))]] = True
        return m
    M["topk_ties_to_higher_index"] = ("topk_mask", topk_ties_high)

    def ranks_flipped(score):
        s = np.asarray(score, np.float64)
        n = s.size
        order = np.lexsort((np.arange(n), -s))
        R = np.empty(n, np.int64)
        R[order] = np.arange(n) + 1
        return R
    M["glass_rank_direction_flipped"] = ("glass_ranks", ranks_flipped)

    M["glass_lambda_swapped"] = ("glass_fuse", lambda Rl, Rg, lam:
                                 lam * np.asarray(Rl, np.float64) + (1 - lam) * np.asarray(Rg, np.float64))

    M["gemv_ignores_mask"] = ("masked_gemv", lambda x, mask, W:
                              np.atleast_2d(np.asarray(x, np.float64)) @ np.asarray(W, np.float64))

    def gemv_union_mask(x, mask, W):
        x = np.atleast_2d(np.asarray(x, np.float64))
        m = np.atleast_2d(np.asarray(mask, bool)).any(axis=0, keepdims=True)
        return (x * m) @ np.asarray(W, np.float64)
    M["gemv_applies_union_mask"] = ("masked_gemv", gemv_union_mask)

    M["silu_drops_factor_v"] = ("silu", lambda v: 1.0 / (1.0 + np.exp(-np.asarray(v, np.float64))))
    M["gelu_is_tanh_form"] = ("gelu_erf", O.gelu_tanh)

    def swiglu_silu_on_up(x, t_in, W_g, W_u, W_d, t_h):
        x = np.atleast_2d(np.asarray(x, np.float64))
        m_x = O.magnitude_mask(x, t_in)
        g = O.masked_gemv(x, m_x, W_g)
        u = O.masked_gemv(x, m_x, W_u)
        h = g * O.silu(u)
        m_h = O.magnitude_mask(h, t_h)
        return O.masked_gemv(h, m_h, W_d), h, m_x, m_h
    M["swiglu_silu_on_up"] = ("ffn_swiglu", swiglu_silu_on_up)

    def route_no_renorm(logits, top_k, renormalize=True):
        return O.__dict__["_orig_moe_route"](logits, top_k, False)
    M["route_not_renormalised"] = ("moe_route", route_no_renorm)

    def expert_mask_on_gate(x, W_g, W_upT, W_d, t_e):
        x = np.asarray(x, np.float64)
        gate = x @ np.asarray(W_g, np.float64)
        a = O.silu(gate)
        m = np.abs(gate) > t_e
        u = np.asarray(W_upT, np.float64) @ x
        return np.where(m, a * u, 0.0) @ np.asarray(W_d, np.float64), a, m
    M["expert_mask_on_raw_gate"] = ("moe_expert", expert_mask_on_gate)

    def layer_no_shared(x, logits, W_g, W_upT, W_d, t_e, top_k, Ws_g=None, Ws_u=None, Ws_d=None,
                        renormalize=True):
        return O.__dict__["_orig_moe_layer"](x, logits, W_g, W_upT, W_d, t_e, top_k, None, None, None,
                                             renormalize)
    M["layer_drops_shared_expert"] = ("moe_layer", layer_no_shared)

    M["gxo_not_rounded_to_fp32"] = ("gxo_score", lambda g, h: np.abs(
        np.asarray(g, np.float64) * np.asarray(h, np.float64)))

    M["corrected_gxo_drops_half"] = ("corrected_gxo_score", lambda g, h: (
        np.asarray(g, np.float64) * np.asarray(h, np.float64)
        + np.abs(np.asarray(h, np.float64)) * math.sqrt(float(np.sum(np.asarray(g, np.float64) ** 2)))))

    def cgxo_f32(signed=True, l2=True, half=True):
        def f(g, h):
            g32 = np.asarray(g, np.float32).astype(np.float64)
            h32 = np.asarray(h, np.float32).astype(np.float64)
            n = math.sqrt(math.fsum((g32 * g32).tolist())) if l2 else float(np.sum(np.abs(g32)))
            n = np.float64(np.float32(n)) * (0.5 if half else 1.0)
            t1 = (g32 * h32).astype(np.float32).astype(np.float64)
            if not signed:
                t1 = np.abs(t1)
            t2 = (np.abs(h32) * n).astype(np.float32).astype(np.float64)
            return (t1 + t2).astype(np.float32)
        return f
    M["corrected_f32_ranks_abs_gxo"] = ("corrected_gxo_score_f32", cgxo_f32(signed=False))
    M["corrected_f32_norm_is_l1"] = ("corrected_gxo_score_f32", cgxo_f32(l2=False))
    M["corrected_f32_drops_half"] = ("corrected_gxo_score_f32", cgxo_f32(half=False))

    def static_ignores_mask(x, W_a, W_d, keep, act="gelu", W_b=None):
        return O.__dict__["_orig_ffn_static_mask"](x, W_a, W_d, np.ones_like(np.asarray(keep, bool)),
                                                   act, W_b)
    M["static_ffn_ignores_mask"] = ("ffn_static_mask", static_ignores_mask)

    def round_bf16_truncates(y, dtype):
        if dtype != "bf16":
            return O.__dict__["_orig_round_to"](y, dtype)
        f = np.asarray(y, np.float64).astype(np.float32)
        bits = (f.view(np.uint32) >> 16) << 16
        return bits.astype(np.uint32).view(np.float32).astype(np.float64)
    M["bf16_rounding_truncates"] = ("round_to", round_bf16_truncates)
    def greedy_largest_growth(err, weights, step, target):
        err = np.asarray(err, np.float64)
        M_, P = err.shape
        lvl = np.zeros(M_, np.int64)
        while O.overall_sparsity(lvl * step, weights) < target - 1e-12:
            g = [err[i, lvl[i] + 1] - err[i, lvl[i]] if lvl[i] + 1 < P else -math.inf
                 for i in range(M_)]
            i = int(np.argmax(g))
            if g[i] == -math.inf:
                break
            lvl[i] += 1
        return lvl
    M["greedy_largest_growth"] = ("greedy_allocate", greedy_largest_growth)

    def greedy_raw_growth(err, weights, step, target):
        err = np.asarray(err, np.float64)
        M_, P = err.shape
        lvl = np.zeros(M_, np.int64)
        while O.overall_sparsity(lvl * step, weights) < target - 1e-12:
            g = [err[i, lvl[i] + 1] - err[i, lvl[i]] if lvl[i] + 1 < P else math.inf
                 for i in range(M_)]
            i = int(np.argmin(g))
            if g[i] == math.inf:
                break
            lvl[i] += 1
        return lvl
    M["greedy_raw_growth"] = ("greedy_allocate", greedy_raw_growth)

    M["overall_unweighted"] = ("overall_sparsity",
                               lambda p, weights: float(np.mean(np.asarray(p, np.float64))))

    def block_error_output_norm(X, W, levels):
        X = np.atleast_2d(np.asarray(X, np.float64))
        err, thr = [], []
        for p in levels:
            t = O.calibrate_threshold(X, p)
            err.append(float(np.linalg.norm(O.masked_gemv(X, O.magnitude_mask(X, t), W))))
            thr.append(t)
        return np.array(err), np.array(thr)
    M["block_error_output_norm"] = ("block_error_curve", block_error_output_norm)

    return M


MUTANT_NAMES = [
    "calib_off_by_one", "calib_floor", "mask_non_strict", "topk_ties_to_higher_index",
    "glass_rank_direction_flipped", "glass_lambda_swapped", "gemv_ignores_mask",
    "gemv_applies_union_mask", "silu_drops_factor_v", "gelu_is_tanh_form",
    "swiglu_silu_on_up", "route_not_renormalised", "expert_mask_on_raw_gate",
    "layer_drops_shared_expert", "gxo_not_rounded_to_fp32", "corrected_gxo_drops_half",
    "corrected_f32_ranks_abs_gxo", "corrected_f32_norm_is_l1", "corrected_f32_drops_half",
    "static_ffn_ignores_mask",
    "bf16_rounding_truncates", "greedy_largest_growth", "greedy_raw_growth", "overall_unweighted",
    "block_error_output_norm",
]


def apply(name):
    """Swap the named oracle function (in the module and the package namespace)."""
    import oracle
    import oracle.sfx_oracle as O
    fn_name, fn = _mutants(O)[name]
    O.__dict__["_orig_" + fn_name] = getattr(O, fn_name)
    setattr(O, fn_name, fn)
    setattr(oracle, fn_name, fn)
