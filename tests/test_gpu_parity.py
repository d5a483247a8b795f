"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle.

Masks, index lists, counts and calibrated thresholds are compared bit for bit;
floating-point outputs within rel-L2 <= 1e-3 and max-abs <= 1e-2 max|y| of the
oracle rounded to the output dtype. Inputs come from the seeded generators in
sparse_input_gemv_b200.synth (Laplace activations, N(0, 0.02^2) weights).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from helpers import assert_close, pack_bitmap, to64
from sparse_input_gemv_b200 import binding as sb
from sparse_input_gemv_b200 import synth

pytestmark = pytest.mark.gpu

DT = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    sb.load()
    yield
    ws = sb.default_workspace()
    if ws.buf is not None:
        assert ws.status() == 0, "device status word raised"


def dev(t):
    return t.to("cuda").contiguous()


def weights(K, N, seed_name, dtype, device="cpu"):
    return synth.normal((K, N), synth.seed_of(seed_name, "W"), 0.02, dtype, device=device)


# ---------------------------------------------------------------- calibration

@pytest.mark.parametrize("dtype,S,K,ps", [
    ("f16", 64, 256, [0.5]),                                  # single input-sparse GEMV workload
    ("bf16", 64, 4096, [0.25, 0.40, 0.50, 0.65]),             # Llama-3-8B block inputs
    ("bf16", 16, 1000, [0.0, 0.1, 0.7, 0.9, 1.0]),            # ragged K, p = 0 and p = 1
    ("f32", 64, 768, [0.5, 0.8, 0.9]),                        # fp32 activations (3 radix passes)
])
def test_calibration_bit_exact(dtype, S, K, ps):
    calib = synth.calib_draws("calib-test", f"{dtype}-{K}", S, K, dtype)
    t_gpu = sb.sfx_calibrate_thresholds(dev(calib), ps)
    a = to64(calib)
    for p, tg in zip(ps, t_gpu):
        assert tg == O.calibrate_threshold(a, p), (p, tg)
        if p > 0:
            frac = np.mean(~O.magnitude_mask(a, tg))
            assert frac >= p - 1e-12


def test_threshold_table_calibrates_once_and_reloads(tmp_path):
    from sparse_input_gemv_b200.thresholds import ThresholdTable
    calib = dev(synth.calib_draws("table", "x", 64, 4096, "bf16"))
    ps = [0.0, 0.25, 0.5, 0.9]
    path = str(tmp_path / "table.json")
    tab = ThresholdTable(path)
    t1 = tab.calibrate("cfg", "ffn-in", calib, ps, seed=3)
    assert t1 == sb.sfx_calibrate_thresholds(calib, ps)
    tab.save()
    # a reloaded table answers without the calibration draws
    back = ThresholdTable(path)
    assert back.calibrate("cfg", "ffn-in", None, ps, seed=3) == t1
    assert t1[2] == O.calibrate_threshold(to64(calib.cpu()), 0.5)


def test_calibration_heavy_ties_f32():
    # values on a coarse grid: the order statistic sits inside long runs of ties
    x = torch.from_numpy(np.round(np.random.default_rng(0).laplace(size=(32, 500)) * 4) / 4)
    x = x.to(torch.float32)
    ps = [0.3, 0.55, 0.95]
    t = sb.sfx_calibrate_thresholds(dev(x), ps)
    for p, tg in zip(ps, t):
        assert tg == O.calibrate_threshold(to64(x), p)


# ---------------------------------------------------------------- mask / compaction

def test_teal_worked_example_on_gpu(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "teal_worked_example.json")))
    for dtype in ("f32", "f16"):
        x = torch.tensor([g["x"]], dtype=DT[dtype])
        out = sb.sfx_mask_compact(dev(x), sb.SFX_SEL_THRESHOLD, t=g["threshold"])
        c = int(out["cnt"][0])
        assert c == 2 and out["idx"][0, :c].tolist() == g["active_idx"]
        assert out["bitmap"][0, 0].item() == 0b01010
    # and through the fused GEMV: y = sparse_x W on the stored (fp16) values
    W = weights(5, 8, "worked", "f16")
    x = torch.tensor(g["x"], dtype=torch.float16)
    y, bm = sb.sfx_sparse_gemv(dev(x), dev(W), t=g["threshold"], out_dtype=torch.float32,
                               want_bitmap=True)
    assert bm[0, 0].item() == 0b01010
    sparse_x = to64(x) * np.array(g["mask"])
    assert_close(to64(y), O.round_to(sparse_x @ to64(W), "f32"), "worked")


@pytest.mark.parametrize("dtype,B,K,t", [("bf16", 1, 4096, 0.69), ("f16", 4, 1000, 1.0),
                                         ("f32", 16, 14336, 0.3), ("bf16", 3, 33, 0.5)])
def test_threshold_mask_compact_bit_exact(dtype, B, K, t):
    x = synth.eval_draw("mask-test", f"{dtype}{K}", B, K, dtype)
    out = sb.sfx_mask_compact(dev(x), sb.SFX_SEL_THRESHOLD, t=t, want_union=True)
    m = O.magnitude_mask(to64(x), t)
    assert np.array_equal(out["bitmap"].cpu().numpy(), pack_bitmap(m))
    for b in range(B):
        idx, c = O.compact(m[b])
        assert int(out["cnt"][b]) == c
        assert np.array_equal(out["idx"][b, :c].cpu().numpy(), idx)
    uidx, uc = O.compact(O.union_mask(m))
    assert int(out["union_cnt"][0]) == uc
    assert np.array_equal(out["union_idx"][:uc].cpu().numpy(), uidx)


@pytest.mark.parametrize("K,keep", [(10240, 0.3), (10240, 0.5), (10240, 0.7), (1000, 0.5), (37, 1.0),
                                    (32768, 0.5), (32767, 0.1), (1025, 0.0)])
def test_topk_gxo_bit_exact(K, keep):
    h = synth.normal((1, K), synth.seed_of("gxo", K, "h"), 1.0, "f32")
    g = synth.normal((1, K), synth.seed_of("gxo", K, "g"), 1.0, "f32")
    k = O.keep_count(keep, K)
    out = sb.sfx_mask_compact(dev(h), sb.SFX_SEL_TOPK_GXO, k=k, score_l=dev(g))
    m = O.topk_mask(O.gxo_score(h.numpy()[0], g.numpy()[0]), k)
    assert int(out["cnt"][0]) == k
    assert np.array_equal(out["idx"][0, :k].cpu().numpy(), O.compact(m)[0])
    assert np.array_equal(out["bitmap"].cpu().numpy(), pack_bitmap(m[None]))


@pytest.mark.parametrize("K,keep,xdt", [(10240, 0.3, "f32"), (10240, 0.5, "f32"), (10240, 0.7, "f32"),
                                        (1000, 0.5, "bf16"), (37, 1.0, "f32"), (32768, 0.5, "f16"),
                                        (3001, 0.0, "f32")])
def test_topk_corrected_gxo_bit_exact(K, keep, xdt):
    # ATTR "correction term": signed g h + |h| ||g|| / 2, ranked in float32
    h = synth.normal((1, K), synth.seed_of("cgxo", K, "h"), 1.0, xdt)
    g = synth.normal((1, K), synth.seed_of("cgxo", K, "g"), 1.0, "f32")
    k = O.keep_count(keep, K)
    out = sb.sfx_mask_compact(dev(h), sb.SFX_SEL_TOPK_CGXO, k=k, score_l=dev(g))
    s = O.corrected_gxo_score_f32(g.numpy()[0], to64(h)[0].astype(np.float32))
    m = O.topk_mask(s, k)
    assert int(out["cnt"][0]) == k
    assert np.array_equal(out["idx"][0, :k].cpu().numpy(), O.compact(m)[0])
    assert np.array_equal(out["bitmap"].cpu().numpy(), pack_bitmap(m[None]))


def test_topk_corrected_gxo_ties_and_batch():
    # equal scores everywhere (ties to the lower index) and a second token with
    # its own norm
    K = 2048
    h = torch.ones((2, K), dtype=torch.float32)
    h[1] = torch.linspace(-3, 3, K)
    g = torch.full((2, K), 0.5, dtype=torch.float32)
    g[1, ::7] = -2.0
    for k in (0, 1, 100, 2047, 2048):
        out = sb.sfx_mask_compact(dev(h), sb.SFX_SEL_TOPK_CGXO, k=k, score_l=dev(g))
        for b in range(2):
            m = O.topk_mask(O.corrected_gxo_score_f32(g.numpy()[b], h.numpy()[b]), k)
            assert int(out["cnt"][b]) == k
            assert np.array_equal(out["idx"][b, :k].cpu().numpy(), O.compact(m)[0]), (k, b)


def test_topk_gxo_ties_go_to_lower_index():
    K = 3000
    rng = np.random.default_rng(5)
    h = torch.from_numpy(rng.integers(0, 5, size=(2, K)).astype(np.float32))  # heavy ties
    g = torch.ones((2, K), dtype=torch.float32)
    for k in (0, 1, 17, 1500, 2999, 3000):
        out = sb.sfx_mask_compact(dev(h), sb.SFX_SEL_TOPK_GXO, k=k, score_l=dev(g))
        for b in range(2):
            m = O.topk_mask(O.gxo_score(g.numpy()[b], h.numpy()[b]), k)
            assert int(out["cnt"][b]) == k
            assert np.array_equal(out["idx"][b, :k].cpu().numpy(), O.compact(m)[0]), (k, b)


def test_topk_gxo_stops_after_any_digit_pass():
    # The radix select stops once the bin holding the k-th key is kept whole.
    # 120 scores 2^-j (one key per 11-bit top digit) over zeros stop after the
    # first pass for k <= 120 and tie-break the zeros after three passes above;
    # consecutive floats 1 + j ulp share their top 22 bits in runs of 1024 and
    # stop after two passes or three; a mix of powers and ulps stops after two
    # or three depending on k. Each case against the oracle, bit for bit.
    K = 4096
    j = np.arange(K)
    cases = {
        "powers": np.where(j < 120, np.ldexp(1.0, -np.minimum(j, 119)), 0.0).astype(np.float32),
        "ulps": (np.float32(1.0) + j.astype(np.float32) * np.float32(2.0 ** -23)).astype(np.float32),
        "mixed": np.where(j % 2 == 0, np.ldexp(1.0, -(j % 60)),
                          1.0 + j * 2.0 ** -23).astype(np.float32),
    }
    for name, hv in cases.items():
        h = torch.from_numpy(np.stack([hv, hv[::-1].copy()]))
        g = torch.ones((2, K), dtype=torch.float32)
        for k in (1, 5, 120, 121, 511, 1024, 1025, 2048, 4095):
            out = sb.sfx_mask_compact(dev(h), sb.SFX_SEL_TOPK_GXO, k=k, score_l=dev(g))
            for b in range(2):
                m = O.topk_mask(O.gxo_score(h.numpy()[b], g.numpy()[b]), k)
                assert int(out["cnt"][b]) == k
                assert np.array_equal(out["idx"][b, :k].cpu().numpy(), O.compact(m)[0]), (name, k, b)


@pytest.mark.parametrize("lam,K,keep", [(0.5, 10240, 0.5), (0.0, 2000, 0.3), (1.0, 2000, 0.7),
                                        (0.3, 999, 0.5)])
def test_glass_bit_exact(lam, K, keep):
    sl = synth.abs_normal((1, K), synth.seed_of("glass", K, "local"))
    sg = synth.abs_normal((1, K), synth.seed_of("glass", K, "global"))
    k = O.keep_count(keep, K)
    out = sb.sfx_mask_compact(None, sb.SFX_SEL_TOPK_GLASS, k=k, score_l=dev(sl), score_g=dev(sg),
                              lam=lam)
    m = O.glass_mask(sl.numpy()[0], sg.numpy()[0], lam, k)
    assert int(out["cnt"][0]) == k
    assert np.array_equal(out["idx"][0, :k].cpu().numpy(), O.compact(m)[0])


# ---------------------------------------------------------------- sparse GEMV

def gemv_case(B, K, N, p, wdt="bf16", xdt=None, seed="gemv", flags=0, out="bf16"):
    xdt = xdt or wdt
    calib = synth.calib_draws(seed, f"in{K}", 64, K, xdt)
    t = O.calibrate_threshold(to64(calib), p) if p > 0 else -math.inf
    x = synth.eval_draw(seed, f"in{K}", B, K, xdt)
    W = weights(K, N, f"{seed}{K}x{N}", wdt)
    y, bm = sb.sfx_sparse_gemv(dev(x), dev(W), t=t, out_dtype=DT[out], flags=flags,
                               want_bitmap=True)
    m = O.magnitude_mask(to64(x), t)
    assert np.array_equal(bm.cpu().numpy(), pack_bitmap(m)), "fused mask differs"
    want = O.masked_gemv(to64(x), m, to64(W))
    if flags & sb.SFX_FLAG_GELU:
        want = O.gelu_erf(want)
    assert_close(to64(y), O.round_to(want, out), f"B={B} K={K} N={N} p={p}")
    return y


def test_single_input_sparse_gemv_workload():
    # x fp16 [1 x 256] ~ Laplace, W fp16 [256 x 512] ~ N(0, 0.02^2), t_p for 50%
    gemv_case(1, 256, 512, 0.5, "f16", out="f16")
    gemv_case(1, 256, 512, 0.5, "f16", out="f32")


@pytest.mark.parametrize("K,N,p", [(4096, 6144, 0.5), (4096, 4096, 0.25), (14336, 4096, 0.65),
                                   (4096, 28672, 0.4), (1000, 264, 0.5), (33, 8, 0.5),
                                   (1, 64, 0.0), (5000, 2056, 0.9)])
def test_gemv_b1_shapes(K, N, p):
    gemv_case(1, K, N, p)


def test_gemv_dense_and_empty_limits():
    # p = 0: every row (dense GEMV); p = 1: no row, y = 0
    gemv_case(1, 2048, 1024, 0.0)
    x = synth.eval_draw("lim", "x", 1, 2048, "bf16")
    W = weights(2048, 1024, "lim", "bf16")
    t = float(x.abs().max())
    y = sb.sfx_sparse_gemv(dev(x), dev(W), t=t)
    assert torch.count_nonzero(y).item() == 0


@pytest.mark.parametrize("B,p", [(2, 0.5), (4, 0.5), (8, 0.7), (16, 0.9), (16, 0.3)])
def test_gemv_batch_union(B, p):
    y = gemv_case(B, 4096, 2048, p, seed="union")
    # each token's row equals its batch-1 result
    x = synth.eval_draw("union", "in4096", B, 4096, "bf16")
    calib = synth.calib_draws("union", "in4096", 64, 4096, "bf16")
    t = O.calibrate_threshold(to64(calib), p)
    W = dev(weights(4096, 2048, "union4096x2048", "bf16"))
    for b in (0, B - 1):
        y1 = sb.sfx_sparse_gemv(dev(x[b]), W, t=t)
        assert_close(to64(y[b]), to64(y1), "batch vs single")


def test_gemv_union_mask_flag():
    B, K, N = 4, 1024, 512
    x = synth.eval_draw("umask", "x", B, K, "bf16")
    W = weights(K, N, "umask", "bf16")
    t = 1.2
    y = sb.sfx_sparse_gemv(dev(x), dev(W), t=t, flags=sb.SFX_FLAG_UNION_MASK,
                           out_dtype=torch.float32)
    u = O.union_mask(O.magnitude_mask(to64(x), t))
    want = O.masked_gemv(to64(x), np.broadcast_to(u, (B, K)), to64(W))
    assert_close(to64(y), O.round_to(want, "f32"), "union-mask reading")


def test_gemv_fp16_and_fp32_inputs_and_gelu():
    gemv_case(1, 2560, 10240, 0.0, "f16", out="f32", flags=sb.SFX_FLAG_GELU)
    gemv_case(1, 3000, 1000, 0.5, "bf16", xdt="f32", out="f32")
    gemv_case(2, 3000, 1000, 0.5, "f16", xdt="f32", out="f16")


def test_gemv_index_list_mode():
    K, N = 10240, 2560
    h = synth.normal((K,), synth.seed_of("idx", "h"), 1.0, "f32")
    g = synth.normal((K,), synth.seed_of("idx", "g"), 1.0, "f32")
    W2 = weights(K, N, "idxW2", "f16")
    k = O.keep_count(0.3, K)
    sel = sb.sfx_mask_compact(dev(h), sb.SFX_SEL_TOPK_GXO, k=k, score_l=dev(g))
    y = sb.sfx_sparse_gemv(dev(h), dev(W2), idx=sel["idx"][0], cnt=sel["cnt"],
                           out_dtype=torch.float16)
    want, m = O.ffn_gelu_topk_down(h.numpy(), g.numpy(), to64(W2), k)
    assert_close(to64(y), O.round_to(want, "f16"), "top-k rows")


def test_gemv_bad_index_is_skipped_and_flagged():
    K, N = 512, 256
    x = synth.eval_draw("bad", "x", 1, K, "bf16")[0]
    W = weights(K, N, "bad", "bf16")
    idx = torch.tensor([3, 7, K + 5, 100], dtype=torch.int32)
    cnt = torch.tensor([4], dtype=torch.int32)
    ws = sb.Workspace()
    y = sb.sfx_sparse_gemv(dev(x), dev(W), idx=dev(idx), cnt=dev(cnt), out_dtype=torch.float32,
                           ws=ws)
    assert ws.status() == sb.SFX_DEV_BAD_INDEX
    assert ws.status() == 0  # read-and-clear
    m = np.zeros(K, bool)
    m[[3, 7, 100]] = True
    assert_close(to64(y), O.round_to(O.masked_gemv(to64(x), m, to64(W))[0], "f32"), "bad idx")


# ---------------------------------------------------------------- GEMV on a given mask

@pytest.mark.parametrize("B,K,N,dens,wdt,xdt,flags", [
    (1, 10240, 2560, 0.3, "f16", "f32", 0),          # the Phi-2 down shape, fp32 h
    (2, 1000, 264, 0.5, "bf16", "bf16", 0),           # ragged K (bits past K set) and N
    (5, 4096, 1024, 0.2, "bf16", "bf16", 0),          # 5 tokens stay on CUDA cores
    (3, 2560, 512, 0.4, "f16", "f16", "union"),       # every token on the union's rows
    (1, 777, 128, 0.6, "bf16", "f32", "gelu"),        # epilogue
    (16, 4000, 4096, 0.1, "bf16", "bf16", 0),
])
def test_gemv_given_mask_matches_oracle(B, K, N, dens, wdt, xdt, flags):
    rng = np.random.default_rng(K + B)
    m = rng.random((B, K)) < dens
    words = pack_bitmap(m)
    if K % 32:
        words[:, -1] |= np.int32(-1 << (K % 32))  # bits past K must be ignored
    x = synth.eval_draw("given-mask", f"x{K}", B, K, xdt)
    W = weights(K, N, f"given-mask-{K}", wdt)
    fl = {0: 0, "union": sb.SFX_FLAG_UNION_MASK, "gelu": sb.SFX_FLAG_GELU}[flags]
    y = sb.sfx_sparse_gemv_mask(dev(x), dev(W), dev(torch.from_numpy(words)),
                                out_dtype=torch.float32, flags=fl)
    mm = np.broadcast_to(O.union_mask(m), (B, K)) if flags == "union" else m
    want = O.masked_gemv(to64(x), mm, to64(W))
    if flags == "gelu":
        want = O.gelu_erf(want)
    assert_close(to64(y), O.round_to(want, "f32"), f"given mask B={B} K={K}")


@pytest.mark.parametrize("xdt", ["bf16", "f32"])
def test_gemv_misaligned_x_on_both_mask_paths(xdt):
    # x one element past a 16-byte boundary (a view into a larger buffer): the
    # compaction's vector loads fall back to element loads; the fused threshold
    # and the given mask must still match the oracle
    B, K, N = 1, 3000, 512
    big = synth.eval_draw("misaligned", "x", 1, K + 1, xdt)
    x = dev(big)[:, 1:]  # not 16-byte aligned, still row-contiguous
    assert x.data_ptr() % 16 != 0
    W = weights(K, N, "misaligned", "bf16")
    t = 0.7
    y_t = sb.sfx_sparse_gemv(x, dev(W), t=t, out_dtype=torch.float32)
    m = O.magnitude_mask(to64(big[:, 1:]), t)
    y_m = sb.sfx_sparse_gemv_mask(x, dev(W), dev(torch.from_numpy(pack_bitmap(m))),
                                  out_dtype=torch.float32)
    want = O.masked_gemv(to64(big[:, 1:]), m, to64(W))
    assert_close(to64(y_t), O.round_to(want, "f32"), "threshold, misaligned x")
    assert_close(to64(y_m), O.round_to(want, "f32"), "given mask, misaligned x")


def test_topk_gxo_at_the_largest_batch():
    # 64 tokens (the top-k's limit), one CTA each, every token its own k-th key
    B, K, k = 64, 1500, 333
    h = synth.normal((B, K), synth.seed_of("gxo-b64", "h"), 1.0, "f32")
    g = synth.normal((B, K), synth.seed_of("gxo-b64", "g"), 1.0, "f32")
    out = sb.sfx_mask_compact(dev(h), sb.SFX_SEL_TOPK_GXO, k=k, score_l=dev(g))
    for b in range(B):
        m = O.topk_mask(O.gxo_score(h.numpy()[b], g.numpy()[b]), k)
        assert int(out["cnt"][b]) == k
        assert np.array_equal(out["idx"][b, :k].cpu().numpy(), O.compact(m)[0]), b
    assert np.array_equal(out["bitmap"].cpu().numpy(),
                          pack_bitmap(np.stack([O.topk_mask(O.gxo_score(h.numpy()[b], g.numpy()[b]), k)
                                                for b in range(B)])))


def test_gemv_given_mask_at_the_largest_k():
    # K = 49152 rows (beyond one CTA's list capacity at one split: the plan
    # splits K), a sparse mask, fp32 x
    B, K, N = 1, 49152, 256
    x = synth.eval_draw("given-mask-bigk", "x", B, K, "f32")
    W = weights(K, N, "given-mask-bigk", "bf16")
    m = np.random.default_rng(9).random((B, K)) < 0.05
    y = sb.sfx_sparse_gemv_mask(dev(x), dev(W), dev(torch.from_numpy(pack_bitmap(m))),
                                out_dtype=torch.float32)
    assert_close(to64(y), O.round_to(O.masked_gemv(to64(x), m, to64(W)), "f32"), "K = 49152")


def test_gemv_given_mask_empty_and_full():
    B, K, N = 2, 3000, 256
    x = synth.eval_draw("given-mask-ef", "x", B, K, "bf16")
    W = weights(K, N, "given-mask-ef", "bf16")
    zero = torch.zeros((B, (K + 31) // 32), dtype=torch.int32)
    y0 = sb.sfx_sparse_gemv_mask(dev(x), dev(W), dev(zero), out_dtype=torch.float32)
    assert torch.count_nonzero(y0) == 0
    full = torch.full((B, (K + 31) // 32), -1, dtype=torch.int32)
    y1 = sb.sfx_sparse_gemv_mask(dev(x), dev(W), dev(full), out_dtype=torch.float32)
    y_dense = sb.sfx_sparse_gemv(dev(x), dev(W), t=-math.inf, out_dtype=torch.float32,
                                 flags=sb.SFX_FLAG_CUDA_CORES)
    assert torch.equal(y1, y_dense)  # same plan, same split order: the same bits


def test_gemv_given_mask_equals_its_own_threshold():
    # the fused |x| > t mask, written out and passed back in, gives the same bits
    B, K, N = 2, 8192, 2048
    x = dev(synth.eval_draw("given-mask-t", "x", B, K, "bf16"))
    W = dev(weights(K, N, "given-mask-t", "bf16"))
    y_t, bm = sb.sfx_sparse_gemv(x, W, t=0.8, out_dtype=torch.float32, want_bitmap=True)
    y_m = sb.sfx_sparse_gemv_mask(x, W, bm, out_dtype=torch.float32)
    assert torch.equal(y_t, y_m)


# ---------------------------------------------------------------- SwiGLU FFN

def ffn_case(B, d, ffn, p, dtype="bf16", seed="ffn"):
    calib_x = synth.calib_draws(seed, f"x{d}", 64, d, dtype)
    t_in = O.calibrate_threshold(to64(calib_x), p) if p > 0 else -math.inf
    Wg = weights(d, ffn, f"{seed}-g", dtype, "cuda")
    Wu = weights(d, ffn, f"{seed}-u", dtype, "cuda")
    Wd = weights(ffn, d, f"{seed}-d", dtype, "cuda")
    Wgu = sb.sfx_pack_gate_up(Wg, Wu)
    Wg64, Wu64, Wd64 = to64(Wg), to64(Wu), to64(Wd)
    # down-site threshold: the oracle's dense FFN h on 16 calibration draws
    if p > 0:
        _, hc, _, _ = O.ffn_swiglu(to64(calib_x[:16]), -math.inf, Wg64, Wu64, Wd64, -math.inf)
        t_h = float(np.float32(O.calibrate_threshold(hc, p)))
    else:
        t_h = -math.inf
    x = synth.eval_draw(seed, f"x{d}", B, d, dtype)
    out = sb.sfx_sparse_ffn_swiglu(dev(x), Wgu, Wd, t_in, t_h, want_h=True, want_bitmaps=True)
    y, h, m_x, m_h = O.ffn_swiglu(to64(x), t_in, Wg64, Wu64, Wd64, t_h)
    # stage 1: exact input mask, h (fp32, unrounded) within tolerance
    assert np.array_equal(out["bitmap_x"].cpu().numpy(), pack_bitmap(m_x))
    assert_close(to64(out["h"]), O.round_to(h, "f32"), "h")
    # stage 2: the fused |h| > t_h mask may differ from the fp64 one only where
    # the fp32 and fp64 h straddle t_h, i.e. within rounding distance of t_h
    got_mh = out["bitmap_h"].cpu().numpy()
    want_mh = pack_bitmap(m_h)
    flips = np.flatnonzero(np.unpackbits((got_mh ^ want_mh).view(np.uint8), bitorder="little"))
    flips = flips[flips % (((ffn + 31) // 32) * 32) < ffn]
    hb = np.abs(h).ravel()
    for f in flips:
        b, j = divmod(int(f), ((ffn + 31) // 32) * 32)
        assert abs(abs(h[b, j]) - t_h) <= 1e-4 * hb.max(), (b, j, h[b, j], t_h)
    assert flips.size <= max(2, ffn * B // 1000)
    assert_close(to64(out["y"]), O.round_to(y, dtype), "y (end to end)")
    return int(flips.size)


def test_ffn_swiglu_small_ragged():
    ffn_case(1, 512, 1796, 0.5)
    ffn_case(3, 264, 1000, 0.4, "f16")


@pytest.mark.parametrize("p", [0.25, 0.40, 0.50, 0.65])
def test_ffn_swiglu_llama3_8b(p):
    flips = ffn_case(1, 4096, 14336, p, seed="llama3-8b-ffn")
    assert flips <= 2


def test_ffn_swiglu_dense_equals_p0():
    ffn_case(2, 1024, 2048, 0.0)


def test_workspace_shared_across_operations():
    # One workspace for every call: scratch written by calibration, GLASS and
    # the FFN must never disturb the GEMV's split-K counters in the header.
    ws = sb.Workspace()
    K, N = 2048, 28672   # many column tiles
    for rep in range(2):
        sl = synth.abs_normal((1, 4096), synth.seed_of("ws", "l"))
        sg = synth.abs_normal((1, 4096), synth.seed_of("ws", "g"))
        sb.sfx_mask_compact(None, sb.SFX_SEL_TOPK_GLASS, k=1000, score_l=dev(sl),
                            score_g=dev(sg), ws=ws)
        calib = synth.calib_draws("ws", "c", 64, 768, "f32")
        sb.sfx_calibrate_thresholds(dev(calib), [0.5], ws=ws)
        x = synth.eval_draw("ws", "x", 1, K, "bf16")
        W = weights(K, N, "ws", "bf16")
        y = sb.sfx_sparse_gemv(dev(x), dev(W), t=0.7, out_dtype=torch.float32, ws=ws)
        want = O.masked_gemv(to64(x), O.magnitude_mask(to64(x), 0.7), to64(W))
        assert_close(to64(y), O.round_to(want, "f32"), f"gemv after other ops ({rep})")
    assert ws.status() == 0


# ---------------------------------------------------------------- batch union on tensor cores
# (the tcgen05 kernel; the default mma.sync kernel has its own test file)

@pytest.fixture
def tc_union():
    with sb.plan_overrides(union_kernel=sb.UNION_TCGEN05):
        yield


@pytest.mark.parametrize("B,K,N,p,wdt,xdt,out", [
    (4, 4096, 2048, 0.5, "bf16", "bf16", "bf16"),
    (16, 1000, 264, 0.3, "f16", "f16", "f32"),     # ragged K and N (N % 128 != 0)
    (8, 14336, 4096, 0.65, "bf16", "f32", "bf16"),  # fp32 inputs: hi + lo bf16 split
    (5, 33, 136, 0.0, "bf16", "bf16", "f32"),       # tiny, dense
    (16, 8192, 1024, 0.9, "bf16", "bf16", "bf16"),  # sparse union (1 - 0.9^16 = 81% rows)
])
def test_union_tensor_core_matches_oracle(B, K, N, p, wdt, xdt, out, tc_union):
    gemv_case(B, K, N, p, wdt, xdt=xdt, seed="tc", out=out)


def test_union_tensor_core_equals_cuda_core_path(tc_union):
    B, K, N = 16, 4096, 3072
    x = synth.eval_draw("tc-vs-cc", "x", B, K, "bf16")
    W = dev(weights(K, N, "tc-vs-cc", "bf16"))
    t = 0.9
    y_tc = sb.sfx_sparse_gemv(dev(x), W, t=t, out_dtype=torch.float32)
    y_cc = sb.sfx_sparse_gemv(dev(x), W, t=t, out_dtype=torch.float32,
                              flags=sb.SFX_FLAG_CUDA_CORES)
    assert_close(to64(y_tc), to64(y_cc), "tensor cores vs CUDA cores")


def test_union_tensor_core_epilogues(tc_union):
    gemv_case(4, 2560, 1024, 0.4, "f16", out="f32", flags=sb.SFX_FLAG_GELU, seed="tc-gelu")
    B, K, N = 6, 1024, 512
    x = synth.eval_draw("tc-umask", "x", B, K, "bf16")
    W = weights(K, N, "tc-umask", "bf16")
    y = sb.sfx_sparse_gemv(dev(x), dev(W), t=1.1, flags=sb.SFX_FLAG_UNION_MASK,
                           out_dtype=torch.float32)
    u = O.union_mask(O.magnitude_mask(to64(x), 1.1))
    want = O.masked_gemv(to64(x), np.broadcast_to(u, (B, K)), to64(W))
    assert_close(to64(y), O.round_to(want, "f32"), "tc union-mask reading")


@pytest.mark.parametrize("B", [4, 16])
def test_ffn_swiglu_batched_tensor_cores(B, tc_union):
    ffn_case(B, 1024, 3584, 0.5, seed=f"ffn-b{B}")


def _cols64(W, j0, j1):
    return W[:, j0:j1].float().cpu().numpy().astype(np.float64)


def _oracle_h_chunked(x64, m_x, Wg, Wu, chunk=2048):
    """The oracle's h = SiLU(g) * u over all neurons, column block by column block
    (the same fp64 products as O.ffn_swiglu without holding all weights in fp64)."""
    xm = np.where(m_x, x64, 0.0)
    ffn = Wg.shape[1]
    h = np.empty((x64.shape[0], ffn))
    for j0 in range(0, ffn, chunk):
        j1 = min(ffn, j0 + chunk)
        g = O.masked_gemv(xm, np.ones_like(m_x), _cols64(Wg, j0, j1))
        u = O.masked_gemv(xm, np.ones_like(m_x), _cols64(Wu, j0, j1))
        h[:, j0:j1] = O.silu(g) * u
    return h


@pytest.mark.parametrize("B", [1, 16])
def test_ffn_swiglu_llama3_70b_full_size_sampled(B):
    # the full 1.4 GB layer in the launch configuration the bench times; the
    # oracle checks the input mask bit for bit, h on every neuron and y on a
    # sample of output columns
    d, ffn, p, seed = 8192, 28672, 0.5, "llama3-70b-ffn"
    calib_x = synth.calib_draws(seed, "x", 64, d, "bf16")
    t_in = O.calibrate_threshold(to64(calib_x), p)
    Wg = weights(d, ffn, f"{seed}-g", "bf16", "cuda")
    Wu = weights(d, ffn, f"{seed}-u", "bf16", "cuda")
    Wd = weights(ffn, d, f"{seed}-d", "bf16", "cuda")
    Wgu = sb.sfx_pack_gate_up(Wg, Wu)
    hc = _oracle_h_chunked(to64(calib_x[:16]), np.ones((16, d), bool), Wg, Wu)
    t_h = float(np.float32(O.calibrate_threshold(hc, p)))
    x = synth.eval_draw(seed, "x", B, d, "bf16")
    out = sb.sfx_sparse_ffn_swiglu(dev(x), Wgu, Wd, t_in, t_h, want_h=True, want_bitmaps=True)
    x64 = to64(x)
    m_x = O.magnitude_mask(x64, t_in)
    assert np.array_equal(out["bitmap_x"].cpu().numpy(), pack_bitmap(m_x))
    h = _oracle_h_chunked(x64, m_x, Wg, Wu)
    assert_close(to64(out["h"]), O.round_to(h, "f32"), "h (70B)")
    m_h = O.magnitude_mask(h, t_h)
    cols = np.sort(np.random.default_rng(17).choice(d, size=256, replace=False))
    Wd_cols = Wd[:, torch.from_numpy(cols).cuda()].float().cpu().numpy().astype(np.float64)
    want = O.masked_gemv(h, m_h, Wd_cols)
    assert_close(to64(out["y"])[:, cols], O.round_to(want, "bf16"), "y sampled columns (70B)")


# ---------------------------------------------------------------- Phi-2 chain end to end

@pytest.mark.parametrize("keep,sel,path", [(0.3, "gxo", "idx"), (0.5, "gxo", "idx"),
                                           (0.7, "gxo", "idx"), (0.3, "cgxo", "idx"),
                                           (0.3, "gxo", "bitmap"), (0.7, "gxo", "bitmap"),
                                           (0.5, "cgxo", "bitmap")])
def test_phi2_gelu_ffn_chain_end_to_end(keep, sel, path):
    # Phi-2-shaped GeLU FFN at batch 1, fp16: the dense up GEMV with the GeLU
    # epilogue, the GxO (or corrected GxO) top-k on the GPU's own h, then the
    # down GEMV on its index list or on its bitmap (path) -- all three on the
    # GPU, compared with the oracle's
    # own chain (fp64 h, its own top-k). The kept set may differ only where the
    # fp32 and fp64 scores straddle the k-th score ("Attribution-based Sparse
    # Activation in Large Language Models", "implementation": top fraction per
    # layer); the flips are counted and y is within the float tolerance.
    d, f = 2560, 10240
    x = synth.eval_draw("phi2-chain", "x", 1, d, "f16")[0]
    W1 = weights(d, f, "phi2-chain-W1", "f16")
    W2 = weights(f, d, "phi2-chain-W2", "f16")
    g = synth.normal((f,), synth.seed_of("phi2-chain", "g"), 1.0, "f32")
    k = O.keep_count(keep, f)
    h_gpu = sb.sfx_sparse_gemv(dev(x), dev(W1), flags=sb.SFX_FLAG_GELU, out_dtype=torch.float32)
    mode = sb.SFX_SEL_TOPK_GXO if sel == "gxo" else sb.SFX_SEL_TOPK_CGXO
    s = sb.sfx_mask_compact(h_gpu[None], mode, k=k, score_l=dev(g)[None],
                            want_idx=(path == "idx"))
    if path == "idx":
        y = sb.sfx_sparse_gemv(h_gpu, dev(W2), idx=s["idx"][0], cnt=s["cnt"],
                               out_dtype=torch.float16)
    else:
        y = sb.sfx_sparse_gemv_mask(h_gpu, dev(W2), s["bitmap"][0], out_dtype=torch.float16)
    # the oracle's chain on the same x, W1, g, W2
    h = O.gelu_erf(to64(x) @ to64(W1))
    h32 = h.astype(np.float32)
    score = O.gxo_score(g.numpy(), h32) if sel == "gxo" else O.corrected_gxo_score_f32(g.numpy(), h32)
    m = O.topk_mask(score, k)
    got = np.unpackbits(s["bitmap"][0].cpu().numpy().view(np.uint8), bitorder="little")[:f] > 0
    if path == "idx":
        assert np.array_equal(np.flatnonzero(got), s["idx"][0, :int(s["cnt"][0])].cpu().numpy())
    assert int(s["cnt"][0]) == k and int(got.sum()) == k
    flips = int(np.count_nonzero(got != m))
    assert flips <= 4, flips
    assert_close(to64(h_gpu), O.round_to(h, "f32"), "h")
    want = O.masked_gemv(h[None], m[None], to64(W2))[0]
    assert_close(to64(y), O.round_to(want, "f16"), f"y keep={keep} {sel} ({flips} flips)")
