"""fp64 CPU oracle for activation-sparse GEMV / FFN / MoE (test infrastructure only).

Sources (cited by page title and section):

[TEAL]  "TEAL: Training-Free Activation Sparsity in Large Language Models"
        (reading-group slides): slide 6 (CATS mask on SiLU(x W_gate)),
        slide 8 (magnitude threshold t_p chosen on calibration data for a target
        sparsity, applied to block inputs), slide 11 ("Hardware-Aware
        Acceleration": fused mask + sparse GEMV, worked example), slide 15
        (speed-ups vs the dense 1.00x baseline).
[ATTR]  "Attribution-based Sparse Activation in Large Language Models"
        (MLSys 2026 talk notes): section "proposed method" (GxO score
        dF/dx * x), section "correction term" (Corrected GxO, Theorem 5.3),
        section "implementation" (keep the top fraction per layer).
[GLASS] "GLASS: Global-Local Aggregation for inference-time Sparsification"
        (technical summary): section 2.2 "rank aggregation".
[GLOSS] "Activation sparsity (LLM)" glossary page: section "why sparsity
        reduces computation" (a zero intermediate skips the matching W2 row).
[MOE]   "Uncovering Intra-expert Activation Sparsity for Efficient
        Mixture-of-Expert Model Execution" (technical summary): section
        "method" (dense gate projection, O(n) threshold mask, fused up/down
        reading only active neurons; shared experts always on).

Conventions. Inputs arrive as numpy arrays holding the exact stored values
(fp16/bf16 inputs decoded to float64). Weights are stored row-per-input-neuron,
W[i, n] with shape [K x N], so y = x W and dropping input neuron i drops row i.
All sums are fp64 over *every* row (the dense definition of the masked
product, no skipping). Where the pages leave a step open, the reading taken is
stated in the function's docstring.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "calibration_rank", "calibrate_threshold", "magnitude_mask", "compact",
    "union_mask", "topk_mask", "keep_count", "gxo_score", "corrected_gxo_score",
    "corrected_gxo_score_f32", "ffn_static_mask",
    "glass_ranks", "glass_fuse", "glass_mask", "masked_gemv", "silu", "gelu_erf",
    "gelu_tanh", "ffn_swiglu", "ffn_gelu_topk_down",
    "moe_route", "moe_expert", "moe_layer", "block_error_curve", "overall_sparsity",
    "greedy_allocate", "round_to",
]


# ----------------------------------------------------------------------------
# a1. threshold calibration                                     [TEAL] slide 8
# ----------------------------------------------------------------------------

def calibration_rank(p: float, n: int) -> int:
    """1-based rank r = ceil(p * n) of the order statistic that is t_p.

    p * n is formed in double precision; a product within 1e-9 * n of an
    integer is taken as that integer so that decimal sparsities such as 0.7
    give the mathematically intended rank (0.7 * 100 -> 70, not 71).
    """
    v = p * n
    r = round(v)
    if abs(v - r) <= 1e-9 * max(n, 1):
        return int(r)
    return int(math.ceil(v))


def calibrate_threshold(calib_abs: np.ndarray, p: float) -> float:
    """Magnitude threshold t_p for target sparsity p on pooled calibration data.

    [TEAL] slide 8: t_p is picked from calibration activations so that the
    target fraction p of magnitudes is zeroed. The slide's formula is lost, so
    the plainest reading is taken: t_p is the lower empirical p-quantile of the
    pooled magnitudes, inf{a : F(a) >= p} = a_(ceil(p N)) with the sorted
    magnitudes a_(1) <= ... <= a_(N). p = 0 keeps everything (t = -inf).
    With the strict mask |x| > t this zeroes at least a fraction p of the
    calibration magnitudes, and no smaller data value would.
    """
    a = np.sort(np.abs(np.asarray(calib_abs, dtype=np.float64)).ravel())
    if p <= 0.0:
        return -math.inf
    r = calibration_rank(p, a.size)
    r = min(max(r, 1), a.size)
    return float(a[r - 1])


# ----------------------------------------------------------------------------
# a3/a4. masks and compaction                       [TEAL] slides 8 and 11
# ----------------------------------------------------------------------------

def magnitude_mask(x: np.ndarray, t: float) -> np.ndarray:
    """m_i = 1[|x_i| > t] ([TEAL] slide 11 worked example; strict inequality)."""
    return np.abs(np.asarray(x, dtype=np.float64)) > t


def compact(mask: np.ndarray):
    """Ascending int32 list of the set positions of a 1-D mask, and its count."""
    idx = np.flatnonzero(np.asarray(mask, dtype=bool)).astype(np.int32)
    return idx, int(idx.size)


def union_mask(masks: np.ndarray) -> np.ndarray:
    """OR over the batch of per-token masks [B x K] -> [K] (the rows to fetch)."""
    return np.any(np.asarray(masks, dtype=bool), axis=0)


def keep_count(keep_fraction: float, n: int) -> int:
    """k = floor(keep * n + 1/2): neurons kept at activation ratio `keep`."""
    return int(math.floor(keep_fraction * n + 0.5))


def topk_mask(score: np.ndarray, k: int) -> np.ndarray:
    """Keep the k largest scores; equal scores are broken toward the lower index.

    [ATTR] "implementation": the top fraction of neurons of a layer by score is
    kept (the per-layer rule). The tie rule (score descending, then index
    ascending) is this library's reading; the pages do not fix one.
    """
    s = np.asarray(score, dtype=np.float64)
    n = s.size
    order = np.lexsort((np.arange(n), -s))  # primary: -s ascending; then index
    m = np.zeros(n, dtype=bool)
    m[order[:max(0, min(k, n))]] = True
    return m


def gxo_score(g: np.ndarray, h: np.ndarray) -> np.ndarray:
    """Attribution score s_j = |g_j * h_j| as a float32 value.

    [ATTR] "proposed method": gradient x output, dF/dx_j * x_j; the magnitude is
    used for ranking. g and h are float32 inputs, so their product is exact in
    float64 and one rounding to float32 gives the correctly rounded float32
    product (the precision the scores are stored in).
    """
    prod = np.asarray(g, dtype=np.float64) * np.asarray(h, dtype=np.float64)
    return np.abs(prod.astype(np.float32))


def corrected_gxo_score(g: np.ndarray, h: np.ndarray) -> np.ndarray:
    """Corrected GxO: g_j h_j + (1/2) |h_j| * ||g||_2  (fp64).

    [ATTR] "correction term": the first term is plain GxO, the second bounds
    the inter-layer attribution error (Theorem 5.3) scaled by 1/2. Pinned by
    closed forms; ``corrected_gxo_score_f32`` is the stored-precision twin the
    GPU selection is compared with.
    """
    g = np.asarray(g, dtype=np.float64)
    h = np.asarray(h, dtype=np.float64)
    return g * h + 0.5 * np.abs(h) * math.sqrt(float(np.sum(g * g)))


def corrected_gxo_score_f32(g: np.ndarray, h: np.ndarray) -> np.ndarray:
    """Corrected GxO in the precision scores are stored and ranked in (float32).

    [ATTR] "correction term": s_j = g_j h_j + (1/2) |h_j| ||g||_2, the norm
    taken over all N1 neurons of the layer. Reading (the pages fix no
    precision): as for plain GxO, each score is a float32 value, built from
    correctly rounded float32 operations in a fixed order,
      n  = fl32(sqrt_fp64(sum_k g_k^2))  (each square exact in fp64, the sum
           correctly rounded: math.fsum; sqrt correctly rounded in fp64),
      t1 = fl32(g_j * h_j),  t2 = fl32(|h_j| * (n / 2)),  s_j = fl32(t1 + t2),
    so that a GPU taking the same steps ranks the same values. The sign is
    kept: negative attributions rank lowest.
    """
    g32 = np.asarray(g, dtype=np.float32)
    h32 = np.asarray(h, dtype=np.float32)
    g64 = g32.astype(np.float64)
    n = np.float32(math.sqrt(math.fsum((g64 * g64).tolist())))
    half_n = np.float32(n * np.float32(0.5))  # exact: a power-of-two scaling
    t1 = (g64 * h32.astype(np.float64)).astype(np.float32)
    t2 = (np.abs(h32).astype(np.float64) * np.float64(half_n)).astype(np.float32)
    return (t1.astype(np.float64) + t2.astype(np.float64)).astype(np.float32)


def glass_ranks(score: np.ndarray) -> np.ndarray:
    """Rank R_j in 1..n with the most important neuron ranked n.

    [GLASS] 2.2: importance scores are turned into ranks before fusion and the
    neurons with the *highest* fused score are kept, so a rank must grow with
    importance. Reading: order by (score descending, index ascending); the
    neuron at position q (0-based) gets rank n - q.
    """
    s = np.asarray(score, dtype=np.float64)
    n = s.size
    order = np.lexsort((np.arange(n), -s))
    R = np.empty(n, dtype=np.int64)
    R[order] = n - np.arange(n)
    return R


def glass_fuse(R_local: np.ndarray, R_global: np.ndarray, lam: float) -> np.ndarray:
    """GLASS_j = (1 - lambda) R^(l)_j + lambda R^(g)_j   ([GLASS] 2.2), fp64."""
    lam = float(lam)
    return (1.0 - lam) * np.asarray(R_local, np.float64) + lam * np.asarray(R_global, np.float64)


def glass_mask(score_local: np.ndarray, score_global: np.ndarray, lam: float, k: int) -> np.ndarray:
    """Top-k of the fused GLASS score ([GLASS] 2.2 "selection"), ties to lower index."""
    F = glass_fuse(glass_ranks(score_local), glass_ranks(score_global), lam)
    return topk_mask(F, k)


# ----------------------------------------------------------------------------
# a5/a7. masked product                    [TEAL] slide 11, [GLOSS] "why"
# ----------------------------------------------------------------------------

def masked_gemv(x: np.ndarray, mask: np.ndarray, W: np.ndarray) -> np.ndarray:
    """y[b, n] = sum_i (x[b,i] * m[b,i]) * W[i, n] in fp64, over all K rows.

    [TEAL] slide 11: sparse_x = x * mask, y = sparse_x @ W. Each token keeps its
    own mask; a batch reads the union of rows, which does not change y_b.
    """
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    m = np.atleast_2d(np.asarray(mask, dtype=bool))
    W = np.asarray(W, dtype=np.float64)
    return (x * m) @ W


def silu(v):
    """SiLU(v) = v * sigma(v) = v / (1 + e^-v)."""
    v = np.asarray(v, dtype=np.float64)
    return v / (1.0 + np.exp(-v))


def gelu_erf(v):
    """GeLU(v) = v * Phi(v) = (v / 2) (1 + erf(v / sqrt 2)) (exact form)."""
    v = np.asarray(v, dtype=np.float64)
    erf = np.vectorize(math.erf, otypes=[np.float64])
    return 0.5 * v * (1.0 + erf(v / math.sqrt(2.0)))


def gelu_tanh(v):
    """tanh approximation of GeLU: (v/2)(1 + tanh(sqrt(2/pi)(v + 0.044715 v^3)))."""
    v = np.asarray(v, dtype=np.float64)
    return 0.5 * v * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (v + 0.044715 * v ** 3)))


# ----------------------------------------------------------------------------
# a6. SwiGLU FFN with TEAL sites on the gate/up input and the down input
# ----------------------------------------------------------------------------

def ffn_swiglu(x, t_in, W_g, W_u, W_d, t_h):
    """Activation-sparse SwiGLU FFN for a batch x [B x d].

    [TEAL] slide 8: the block input is masked by |x| > t_in; the down
    projection's input h is masked by |h| > t_h. h = SiLU(g) * u with
    g = (x m_x) W_g, u = (x m_x) W_u. h is kept unrounded (fp64 here).
    Returns (y, h, m_x, m_h).
    """
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    m_x = magnitude_mask(x, t_in)
    g = masked_gemv(x, m_x, W_g)
    u = masked_gemv(x, m_x, W_u)
    h = silu(g) * u
    m_h = magnitude_mask(h, t_h)
    y = masked_gemv(h, m_h, W_d)
    return y, h, m_x, m_h


def ffn_static_mask(x, W_a, W_d, keep, act="gelu", W_b=None):
    """FFN whose intermediate neurons outside a fixed set are pruned on both sides.

    [GLASS] "selection": with a neuron mask fixed for the prompt, the pruned
    neurons' up-projection columns and down-projection rows are both skipped.
    Written as the dense definition: h = act(x W_a) (GeLU, tanh GeLU) or
    SiLU(x W_a) * (x W_b) (SwiGLU), then y = (h * m) W_d. x [B x d],
    W_a / W_b [d x ffn], W_d [ffn x d], keep [ffn] bool. Returns (y, h).
    """
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    a = x @ np.asarray(W_a, dtype=np.float64)
    if act == "gelu":
        h = gelu_erf(a)
    elif act == "gelu_tanh":
        h = gelu_tanh(a)
    elif act == "swiglu":
        h = silu(a) * (x @ np.asarray(W_b, dtype=np.float64))
    else:
        raise ValueError(act)
    m = np.broadcast_to(np.asarray(keep, dtype=bool), h.shape)
    return masked_gemv(h, m, W_d), h


def ffn_gelu_topk_down(h, g, W2, k):
    """GeLU FFN down projection keeping the top-k neurons by |g * h|.

    [ATTR] "implementation": neurons of a layer are ranked by attribution score
    and the top fraction is kept; the deactivated neurons' weights are skipped.
    h is the GeLU output for one token (float32 values), g the seeded gradient.
    Returns (y, mask).
    """
    s = gxo_score(g, h)
    m = topk_mask(s, k)
    return masked_gemv(np.asarray(h, np.float64)[None, :], m[None, :], W2)[0], m


# ----------------------------------------------------------------------------
# a8. MoE: routing + intra-expert masking                              [MOE]
# ----------------------------------------------------------------------------

def moe_route(logits: np.ndarray, top_k: int, renormalize: bool = True):
    """Softmax over the experts' logits, top_k experts by probability.

    Ties between equal probabilities go to the lower expert index. Reading:
    the selected probabilities are renormalised to sum to 1 (the pages say
    only "top-k softmax routing"); `renormalize=False` keeps raw probabilities.
    Returns (experts [top_k] int, weights [top_k] fp64), experts in selection
    order (probability descending).
    """
    z = np.asarray(logits, dtype=np.float64)
    e = np.exp(z - z.max())
    prob = e / e.sum()
    order = np.lexsort((np.arange(prob.size), -prob))[:top_k]
    w = prob[order]
    if renormalize:
        w = w / w.sum()
    return order.astype(np.int64), w


def moe_expert(x, W_g, W_upT, W_d, t_e):
    """One expert on one token with an intra-expert magnitude mask.

    [MOE] "method": the gate projection is computed densely and gives each
    neuron's activation score; a single threshold pass masks it; the up and
    down projections touch only the active neurons. Reading: the score is
    |SiLU(x W_g)| ([TEAL] slide 6, the CATS site) against a per-expert
    threshold t_e, and the expert output is sum_{j active} a_j u_j W_d[j, :]
    with a = SiLU(x W_g) and u_j = W_upT[j, :] . x.
    Returns (y [d], a [ffn], mask [ffn]).
    """
    x = np.asarray(x, dtype=np.float64)
    gate = x @ np.asarray(W_g, np.float64)
    a = silu(gate)
    m = np.abs(a) > t_e
    u = np.asarray(W_upT, np.float64) @ x
    v = np.where(m, a * u, 0.0)
    y = v @ np.asarray(W_d, np.float64)
    return y, a, m


def moe_layer(x, logits, W_g, W_upT, W_d, t_e, top_k, Ws_g=None, Ws_u=None, Ws_d=None,
              renormalize: bool = True):
    """MoE layer output for a batch x [B x d].

    y_t = sum_{e in top_k(t)} w_{t,e} * expert_e(x_t) + shared(x_t); the shared
    expert is a dense SwiGLU FFN that is always on ([MOE] "method": shared
    experts and the router stay as they are). W_g [E x d x ffn],
    W_upT [E x ffn x d], W_d [E x ffn x d], t_e [E].
    """
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    B, d = x.shape
    y = np.zeros((B, d), dtype=np.float64)
    for t in range(B):
        experts, w = moe_route(logits[t], top_k, renormalize)
        for e, we in zip(experts, w):
            ye, _, _ = moe_expert(x[t], W_g[e], W_upT[e], W_d[e], t_e[e])
            y[t] += we * ye
        if Ws_g is not None:
            ys, _, _, _ = ffn_swiglu(x[t:t + 1], -math.inf, Ws_g, Ws_u, Ws_d, -math.inf)
            y[t] += ys[0]
    return y


# ----------------------------------------------------------------------------
# block-wise greedy sparsity allocation                     [TEAL] slide 10
# ----------------------------------------------------------------------------

def block_error_curve(X, W, levels):
    """l2 activation error of one block at each sparsity level.

    [TEAL] slide 10 optimises the per-block sparsities against the blocks' l2
    activation error. Reading: a block is one input site with its weight
    matrix W [K x N]; at level p its input is masked with the threshold t_p
    calibrated on the same draws X [S x K] (calibrate_threshold), and the
    error is the l2 (Frobenius) norm over the S draws of the change in the
    block output, ||(X * m_p) W - X W||. Returns (err [P], t [P]) in fp64.
    """
    X = np.atleast_2d(np.asarray(X, dtype=np.float64))
    W = np.asarray(W, dtype=np.float64)
    dense = masked_gemv(X, np.ones_like(X, dtype=bool), W)
    err, thr = [], []
    for p in levels:
        t = calibrate_threshold(X, p)
        y = masked_gemv(X, magnitude_mask(X, t), W)
        err.append(float(np.linalg.norm(y - dense)))
        thr.append(t)
    return np.array(err), np.array(thr)


def overall_sparsity(p, weights):
    """Model-wide sparsity of per-block sparsities p: sum_i w_i p_i / sum_i w_i.

    Reading of [TEAL] slide 10's overall sparsity constraint: each block counts
    by its weight w_i, its parameter count, since a block at sparsity p skips
    that fraction of its weight rows (weights of 1 give the plain mean).
    """
    p = np.asarray(p, dtype=np.float64)
    w = np.asarray(weights, dtype=np.float64)
    return float((w * p).sum() / w.sum())


def greedy_allocate(err, weights, step, target):
    """Per-block sparsity levels by [TEAL] slide 10's greedy procedure.

    err [M x P]: block i's error at sparsity level j (levels 0, step, 2 step,
    ..., so err[:, 0] is the dense block). Steps of the slide: every block
    starts at sparsity 0; each round measures, for every block that can still
    go one level up, how much its error would grow; the block whose error
    grows least goes up one level (equal growths: the lower block index);
    rounds repeat until the overall sparsity (overall_sparsity with `weights`)
    reaches `target`, or no block can go further. Reading: blocks of unequal
    weight buy unequal amounts of overall sparsity with one level, so the
    growth is compared per unit of overall sparsity gained, growth / w_i
    (with equal weights this is the raw growth the slide compares). Returns
    the level index of each block (sparsity = level * step).
    """
    err = np.asarray(err, dtype=np.float64)
    w = np.asarray(weights, dtype=np.float64)
    M, P = err.shape
    lvl = np.zeros(M, dtype=np.int64)
    while overall_sparsity(lvl * step, w) < target - 1e-12:
        best, best_i = math.inf, -1
        for i in range(M):
            if lvl[i] + 1 < P and w[i] > 0:
                growth = (err[i, lvl[i] + 1] - err[i, lvl[i]]) / w[i]
                if growth < best:
                    best, best_i = growth, i
        if best_i < 0:
            break
        lvl[best_i] += 1
    return lvl


# ----------------------------------------------------------------------------
# output rounding for comparisons
# ----------------------------------------------------------------------------

def round_to(y: np.ndarray, dtype: str) -> np.ndarray:
    """Round fp64 values to the output dtype (RNE) and back to fp64.

    fp16 uses numpy's float16 cast (RNE from fp64). bf16 and f32 round the fp64
    value to float32 first, then bf16 applies RNE on the float32 bits; the
    double rounding fp64 -> f32 -> bf16 can differ from a direct rounding only
    when the value lies within 2^-24 relative of a bf16 tie, far below the
    comparison tolerance.
    """
    y = np.asarray(y, dtype=np.float64)
    if dtype == "f16":
        return y.astype(np.float16).astype(np.float64)
    f = y.astype(np.float32)
    if dtype == "f32":
        return f.astype(np.float64)
    if dtype == "bf16":
        bits = f.view(np.uint32).astype(np.uint64)
        lsb = (bits >> 16) & 1
        rounded = ((bits + 0x7FFF + lsb) >> 16) << 16
        return rounded.astype(np.uint32).view(np.float32).astype(np.float64)
    raise ValueError(dtype)
