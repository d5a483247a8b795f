"""Thin ctypes binding of libsfx.so (include/sfx.h), with the C ABI's names.

Only argument marshalling happens here: tensors become device pointers, the
current torch stream becomes the cudaStream_t, outputs and workspaces are
allocated with torch (the library itself never allocates). Every step of the
computation runs in the library's CUDA kernels; if libsfx.so is missing or a
call fails, an exception is raised -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsfx.so")

SFX_F16, SFX_BF16, SFX_F32 = 0, 1, 2
SFX_SEL_THRESHOLD, SFX_SEL_TOPK_GXO, SFX_SEL_TOPK_GLASS, SFX_SEL_TOPK_CGXO = 0, 1, 2, 3
SFX_OP_CALIBRATE, SFX_OP_MASK_COMPACT, SFX_OP_SPARSE_GEMV, SFX_OP_FFN_SWIGLU, SFX_OP_MOE, \
    SFX_OP_STATIC_FFN, SFX_OP_ERROR_CURVE = range(7)
SFX_FLAG_GELU, SFX_FLAG_GELU_TANH, SFX_FLAG_UNION_MASK, SFX_FLAG_NO_RENORM, SFX_FLAG_CUDA_CORES = \
    0x1, 0x2, 0x4, 0x8, 0x10
SFX_FLAG_SWIGLU = 0x20
SFX_DEV_BAD_INDEX, SFX_DEV_TIMEOUT = 0x1, 0x2

_DT = {torch.float16: SFX_F16, torch.bfloat16: SFX_BF16, torch.float32: SFX_F32}
_TORCH_DT = {v: k for k, v in _DT.items()}

# (name, restype, argtypes); c_void_p for every pointer, c_longlong for sizes.
_VP, _I, _LL, _F, _D, _SZ = (ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float,
                             ctypes.c_double, ctypes.c_size_t)
_SIGS = {
    "sfx_workspace_bytes": (_SZ, [_I, _LL, _LL, _LL, _LL, _LL, _LL]),
    "sfx_workspace_init": (_I, [_VP, _SZ, _VP]),
    "sfx_status_string": (ctypes.c_char_p, [_I]),
    "sfx_check_device_status": (_I, [_VP, _VP, _VP]),
    "sfx_device_sm_count": (_I, []),
    "sfx_build_info": (ctypes.c_char_p, []),
    "sfx_gemv_plan": (_I, [_I, _LL, _LL, _I, _I, _VP]),
    "sfx_set_plan_override": (_I, [_I, _I]),
    "sfx_set_wait_limit_ns": (_I, [ctypes.c_ulonglong]),
    "sfx_block_error_curve": (_I, [_VP, _I, _LL, _LL, _VP, _I, _LL, _VP, _I, _VP, _VP, _VP, _SZ,
                                   _VP]),
    "sfx_greedy_allocate": (_I, [_VP, _VP, _I, _I, _D, _D, _VP]),
    "sfx_calibrate_thresholds": (_I, [_VP, _I, _LL, _LL, _VP, _I, _VP, _VP, _SZ, _VP]),
    "sfx_mask_compact": (_I, [_VP, _I, _I, _I, _I, _F, _I, _VP, _VP, _D, _VP, _VP, _VP, _VP, _VP,
                              _VP, _SZ, _VP]),
    "sfx_sparse_gemv": (_I, [_VP, _I, _I, _I, _VP, _I, _I, _F, _VP, _VP, _VP, _I, _I, _VP, _VP,
                             _SZ, _VP]),
    "sfx_sparse_gemv_noalloc": (_I, [_VP, _I, _I, _I, _VP, _I, _I, _F, _VP, _VP, _VP, _I, _I,
                                     _VP]),
    "sfx_sparse_gemv_mask": (_I, [_VP, _I, _I, _I, _VP, _I, _I, _VP, _VP, _I, _I, _VP, _SZ, _VP]),
    "sfx_sparse_ffn_swiglu": (_I, [_VP, _I, _I, _I, _I, _VP, _VP, _F, _F, _VP, _I, _VP, _VP, _VP,
                                   _I, _VP, _SZ, _VP]),
    "sfx_pack_gate_up": (_I, [_VP, _VP, _I, _I, _I, _VP, _VP]),
    "sfx_moe_expert_sparse": (_I, [_VP, _I, _VP, _I, _I, _I, _I, _I, _VP, _VP, _VP, _VP, _VP, _VP,
                                   _VP, _I, _VP, _I, _VP, _VP, _I, _VP, _SZ, _VP]),
    "sfx_static_ffn": (_I, [_VP, _I, _I, _I, _I, _VP, _VP, _VP, _VP, _VP, _I, _VP, _I, _VP, _SZ,
                            _VP]),
}
EXPORTED = tuple(_SIGS)

_lib = None


class SfxError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        msg = _lib.sfx_status_string(status).decode() if _lib is not None else str(status)
        super().__init__(f"{fn} failed: {msg} ({status})")


def load(path: str = LIB_PATH):
    """Load libsfx.so (raises if it is missing: build it with build.py)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing; run `python -m sparse_input_gemv_b200.build` "
                           "(the CUDA library is required, there is no CPU fallback)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn, rc):
    if rc != 0:
        raise SfxError(fn, rc)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors passed to the CUDA library must be contiguous CUDA tensors")


# ---------------------------------------------------------------- workspace

def sfx_workspace_bytes(op: int, a=0, b=0, c=0, d=0, e=0, f=0) -> int:
    return int(load().sfx_workspace_bytes(op, a, b, c, d, e, f))


class Workspace:
    """A caller-owned, zero-initialised device workspace that grows on demand.

    Allocate it (``reserve``) before capturing a CUDA graph: a growth inside a
    capture would allocate memory.
    """

    def __init__(self, device=None):
        self.device = torch.device(device or "cuda")
        self.buf = None

    def reserve(self, nbytes: int):
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.device)
            _check("sfx_workspace_init", load().sfx_workspace_init(
                _ptr(self.buf), self.buf.numel(), _stream()))
        return self.buf

    def status(self) -> int:
        """Synchronise, read and clear the device status word (0 = clean)."""
        bits = ctypes.c_uint(0)
        load().sfx_check_device_status(_ptr(self.buf), ctypes.byref(bits), _stream())
        return int(bits.value)


_default_ws = {}


def _ws(ws, nbytes, device):
    if ws is None:
        key = torch.device(device).index if torch.device(device).index is not None else \
            torch.cuda.current_device()
        ws = _default_ws.setdefault(key, Workspace(torch.device("cuda", key)))
    buf = ws.reserve(nbytes)
    return ws, buf


def default_workspace(device=None) -> Workspace:
    dev = torch.device(device or "cuda")
    key = dev.index if dev.index is not None else torch.cuda.current_device()
    return _default_ws.setdefault(key, Workspace(torch.device("cuda", key)))


# ---------------------------------------------------------------- entry points

def sfx_calibrate_thresholds(calib: torch.Tensor, sparsities, ws: Workspace | None = None):
    """t_p for each target sparsity p (host floats); calib is [S x K] on the GPU."""
    _need_cuda(calib)
    S, K = calib.shape
    P = len(sparsities)
    nbytes = sfx_workspace_bytes(SFX_OP_CALIBRATE, S, K, P, _DT[calib.dtype])
    ws, buf = _ws(ws, nbytes, calib.device)
    sp = (ctypes.c_double * P)(*[float(p) for p in sparsities])
    out = (ctypes.c_float * P)()
    _check("sfx_calibrate_thresholds", load().sfx_calibrate_thresholds(
        _ptr(calib), _DT[calib.dtype], S, K, ctypes.cast(sp, ctypes.c_void_p), P,
        ctypes.cast(out, ctypes.c_void_p), _ptr(buf), buf.numel(), _stream()))
    return [float(v) for v in out]


def sfx_mask_compact(x=None, sel=SFX_SEL_THRESHOLD, t=0.0, k=0, score_l=None, score_g=None,
                     lam=0.5, want_union=False, ws: Workspace | None = None, K=None, B=None,
                     want_idx=True):
    """Masks, ascending index lists and counts. Returns dict(bitmap, idx, cnt[, union_idx, union_cnt]);
    idx is None with want_idx=False (the bitmap and counts only)."""
    ref = x if x is not None else score_l
    _need_cuda(x, score_l, score_g)
    if ref.dim() == 1:
        ref = ref[None]
    B_, K_ = ref.shape
    B = B or B_
    K = K or K_
    dev = ref.device
    words = (K + 31) // 32
    bitmap = torch.zeros((B, words), dtype=torch.int32, device=dev)
    idx = torch.full((B, K), -1, dtype=torch.int32, device=dev) if want_idx else None
    cnt = torch.zeros((B,), dtype=torch.int32, device=dev)
    uidx = torch.full((K,), -1, dtype=torch.int32, device=dev) if want_union else None
    ucnt = torch.zeros((1,), dtype=torch.int32, device=dev) if want_union else None
    dt = _DT[x.dtype] if x is not None else SFX_F32
    ws, buf = _ws(ws, sfx_workspace_bytes(SFX_OP_MASK_COMPACT, B, K, sel), dev)
    _check("sfx_mask_compact", load().sfx_mask_compact(
        _ptr(x), dt, B, K, sel, float(t), int(k), _ptr(score_l), _ptr(score_g), float(lam),
        _ptr(bitmap), _ptr(idx), _ptr(cnt), _ptr(uidx), _ptr(ucnt), _ptr(buf), buf.numel(),
        _stream()))
    out = {"bitmap": bitmap, "idx": idx, "cnt": cnt}
    if want_union:
        out["union_idx"], out["union_cnt"] = uidx, ucnt
    return out


def sfx_sparse_gemv(x, W, t=-math.inf, idx=None, cnt=None, out_dtype=None, flags=0,
                    want_bitmap=False, y=None, ws: Workspace | None = None, stream=None):
    """y = (x * m) W reading only active rows of W. x [B x K] (or [K]), W [K x N]."""
    squeeze = x.dim() == 1
    x2 = x[None] if squeeze else x
    _need_cuda(x2, W, idx, cnt)
    B, K = x2.shape
    K2, N = W.shape
    if K2 != K:
        raise ValueError("x and W disagree on K")
    out_dtype = out_dtype or W.dtype
    if flags & SFX_FLAG_SWIGLU:
        out_dtype = torch.float32
    if y is None:
        ncol = N // 2 if flags & SFX_FLAG_SWIGLU else N
        y = torch.empty((B, ncol), dtype=out_dtype, device=W.device)
    bitmap = torch.zeros((B, (K + 31) // 32), dtype=torch.int32, device=W.device) \
        if want_bitmap else None
    ws, buf = _ws(ws, sfx_workspace_bytes(SFX_OP_SPARSE_GEMV, B, K, N, _DT[x2.dtype]), W.device)
    _check("sfx_sparse_gemv", load().sfx_sparse_gemv(
        _ptr(x2), _DT[x2.dtype], B, K, _ptr(W), _DT[W.dtype], N, float(t), _ptr(idx), _ptr(cnt),
        _ptr(y), _DT[y.dtype], int(flags), _ptr(bitmap), _ptr(buf), buf.numel(), _stream(stream)))
    y_out = y[0] if squeeze else y
    return (y_out, bitmap) if want_bitmap else y_out


def sfx_sparse_gemv_mask(x, W, mask, out_dtype=None, flags=0, y=None,
                         ws: Workspace | None = None, stream=None):
    """y = (x * m) W for a given mask bitmap m ([B x ceil(K/32)] int32/uint32 words)."""
    squeeze = x.dim() == 1
    x2 = x[None] if squeeze else x
    mask2 = mask[None] if mask.dim() == 1 else mask
    _need_cuda(x2, W, mask2)
    B, K = x2.shape
    K2, N = W.shape
    if K2 != K:
        raise ValueError("x and W disagree on K")
    if tuple(mask2.shape) != (B, (K + 31) // 32) or mask2.element_size() != 4 \
            or not mask2.is_contiguous():
        raise ValueError("mask must be a contiguous [B x ceil(K/32)] tensor of 32-bit words")
    out_dtype = out_dtype or W.dtype
    if flags & SFX_FLAG_SWIGLU:
        out_dtype = torch.float32
    if y is None:
        ncol = N // 2 if flags & SFX_FLAG_SWIGLU else N
        y = torch.empty((B, ncol), dtype=out_dtype, device=W.device)
    ws, buf = _ws(ws, sfx_workspace_bytes(SFX_OP_SPARSE_GEMV, B, K, N, _DT[x2.dtype]), W.device)
    _check("sfx_sparse_gemv_mask", load().sfx_sparse_gemv_mask(
        _ptr(x2), _DT[x2.dtype], B, K, _ptr(W), _DT[W.dtype], N, _ptr(mask2), _ptr(y),
        _DT[y.dtype], int(flags), _ptr(buf), buf.numel(), _stream(stream)))
    return y[0] if squeeze else y


def sfx_sparse_gemv_noalloc(x, W, t=-math.inf, idx=None, cnt=None, out_dtype=None, flags=0,
                            y=None, stream=None):
    """sfx_sparse_gemv for callers that cannot allocate device memory.

    The library keeps this call's scratch in a fixed 4 MiB device array of its
    own, so only inputs and outputs are passed (``y`` may be preallocated by
    the caller; if it is None this wrapper allocates it with torch, which the
    C entry point itself never does). Calls must not overlap on the GPU.
    """
    squeeze = x.dim() == 1
    x2 = x[None] if squeeze else x
    _need_cuda(x2, W, idx, cnt)
    B, K = x2.shape
    K2, N = W.shape
    if K2 != K:
        raise ValueError("x and W disagree on K")
    out_dtype = torch.float32 if flags & SFX_FLAG_SWIGLU else (out_dtype or W.dtype)
    if y is None:
        y = torch.empty((B, N // 2 if flags & SFX_FLAG_SWIGLU else N), dtype=out_dtype,
                        device=W.device)
    _check("sfx_sparse_gemv_noalloc", load().sfx_sparse_gemv_noalloc(
        _ptr(x2), _DT[x2.dtype], B, K, _ptr(W), _DT[W.dtype], N, float(t), _ptr(idx), _ptr(cnt),
        _ptr(y), _DT[y.dtype], int(flags), _stream(stream)))
    return y[0] if squeeze else y


def sfx_pack_gate_up(W_g, W_u, stream=None):
    """[d x ffn] gate and up weights -> interleaved [d x 2 ffn] (row i: g0 u0 g1 u1 ...)."""
    _need_cuda(W_g, W_u)
    d, ffn = W_g.shape
    W_gu = torch.empty((d, 2 * ffn), dtype=W_g.dtype, device=W_g.device)
    _check("sfx_pack_gate_up", load().sfx_pack_gate_up(
        _ptr(W_g), _ptr(W_u), _DT[W_g.dtype], d, ffn, _ptr(W_gu), _stream(stream)))
    return W_gu


def sfx_sparse_ffn_swiglu(x, W_gu, W_d, t_in=-math.inf, t_h=-math.inf, out_dtype=None, flags=0,
                          want_h=False, want_bitmaps=False, y=None, h=None,
                          ws: Workspace | None = None, stream=None):
    """Activation-sparse SwiGLU FFN; returns y (and h / bitmaps when asked)."""
    squeeze = x.dim() == 1
    x2 = x[None] if squeeze else x
    _need_cuda(x2, W_gu, W_d)
    B, d = x2.shape
    ffn = W_d.shape[0]
    dev = W_d.device
    out_dtype = out_dtype or W_d.dtype
    if y is None:
        y = torch.empty((B, d), dtype=out_dtype, device=dev)
    if want_h and h is None:
        h = torch.empty((B, ffn), dtype=torch.float32, device=dev)
    bx = torch.zeros((B, (d + 31) // 32), dtype=torch.int32, device=dev) if want_bitmaps else None
    bh = torch.zeros((B, (ffn + 31) // 32), dtype=torch.int32, device=dev) if want_bitmaps else None
    ws, buf = _ws(ws, sfx_workspace_bytes(SFX_OP_FFN_SWIGLU, B, d, ffn, _DT[x2.dtype]), dev)
    _check("sfx_sparse_ffn_swiglu", load().sfx_sparse_ffn_swiglu(
        _ptr(x2), _DT[x2.dtype], B, d, ffn, _ptr(W_gu), _ptr(W_d), float(t_in), float(t_h),
        _ptr(y), _DT[y.dtype], _ptr(h), _ptr(bx), _ptr(bh), int(flags), _ptr(buf), buf.numel(),
        _stream(stream)))
    out = {"y": y[0] if squeeze else y}
    if h is not None:
        out["h"] = h
    if want_bitmaps:
        out["bitmap_x"], out["bitmap_h"] = bx, bh
    return out


def sfx_moe_expert_sparse(x, logits, W_gT, W_upT, W_d, t_e, top_k, Ws_gT=None, Ws_upT=None,
                          Ws_d=None, out_dtype=None, flags=0, want_a=False, y=None,
                          ws: Workspace | None = None, stream=None):
    """MoE layer with intra-expert magnitude masks; returns dict(y[, a, sel]).

    W_gT, W_upT, W_d: [E x ffn x d]; the optional shared expert Ws_gT, Ws_upT,
    Ws_d: [ffn_shared x d] (every matrix one row per intermediate neuron).
    """
    squeeze = x.dim() == 1
    x2 = x[None] if squeeze else x
    lg = logits[None] if logits.dim() == 1 else logits
    _need_cuda(x2, lg, W_gT, W_upT, W_d, t_e, Ws_gT, Ws_upT, Ws_d)
    B, d = x2.shape
    E, ffn, _ = W_gT.shape
    W_g = W_gT
    ffn_s = Ws_d.shape[0] if Ws_d is not None else 0
    dev = x2.device
    out_dtype = out_dtype or x2.dtype
    if y is None:
        y = torch.empty((B, d), dtype=out_dtype, device=dev)
    a = torch.empty((B, top_k, ffn), dtype=torch.float32, device=dev) if want_a else None
    sel = torch.empty((B, top_k), dtype=torch.int32, device=dev) if want_a else None
    ws, buf = _ws(ws, sfx_workspace_bytes(SFX_OP_MOE, B, d, E, ffn, top_k, ffn_s), dev)
    _check("sfx_moe_expert_sparse", load().sfx_moe_expert_sparse(
        _ptr(x2), _DT[x2.dtype], _ptr(lg), B, d, E, ffn, top_k, _ptr(W_g), _ptr(W_upT), _ptr(W_d),
        _ptr(t_e), _ptr(Ws_gT), _ptr(Ws_upT), _ptr(Ws_d), ffn_s, _ptr(y), _DT[y.dtype], _ptr(a),
        _ptr(sel),
        int(flags), _ptr(buf), buf.numel(), _stream(stream)))
    out = {"y": y[0] if squeeze else y}
    if want_a:
        out["a"], out["sel"] = a, sel
    return out


def sfx_static_ffn(x, W_aT, W_d, idx, cnt, W_bT=None, flags=0, out_dtype=None, y=None,
                   ws: Workspace | None = None, stream=None):
    """FFN with a static neuron set on both projections; returns y [B x d].

    W_aT (and W_bT for SwiGLU), W_d: [ffn x d] one row per neuron; idx: int32
    kept neurons, cnt: int32 [1] device count; flags: SFX_FLAG_GELU_TANH for
    the tanh GeLU (erf GeLU otherwise; W_bT selects SwiGLU).
    """
    squeeze = x.dim() == 1
    x2 = x[None] if squeeze else x
    _need_cuda(x2, W_aT, W_bT, W_d, idx, cnt)
    B, d = x2.shape
    ffn = W_aT.shape[0]
    if y is None:
        y = torch.empty((B, d), dtype=out_dtype or x2.dtype, device=x2.device)
    ws, buf = _ws(ws, sfx_workspace_bytes(SFX_OP_STATIC_FFN, B, d, ffn), x2.device)
    _check("sfx_static_ffn", load().sfx_static_ffn(
        _ptr(x2), _DT[x2.dtype], B, d, ffn, _ptr(W_aT), _ptr(W_bT), _ptr(W_d), _ptr(idx), _ptr(cnt),
        int(flags), _ptr(y), _DT[y.dtype], _ptr(buf), buf.numel(), _stream(stream)))
    return y[0] if squeeze and y.dim() == 2 else y


def sfx_block_error_curve(calib, W, levels, ws: Workspace | None = None, stream=None):
    """A block's l2 output error at each sparsity level (TEAL slide 10).

    calib [S x K] (GPU, the site's calibration draws), W [K x N] (GPU).
    Returns (err: list of floats, thresholds: list of floats)."""
    _need_cuda(calib, W)
    S, K = calib.shape
    K2, N = W.shape
    if K2 != K:
        raise ValueError("calib and W disagree on K")
    P = len(levels)
    nbytes = sfx_workspace_bytes(SFX_OP_ERROR_CURVE, S, K, N, _DT[calib.dtype], P)
    ws, buf = _ws(ws, nbytes, calib.device)
    lv = (ctypes.c_double * P)(*[float(p) for p in levels])
    err = (ctypes.c_double * P)()
    thr = (ctypes.c_float * P)()
    _check("sfx_block_error_curve", load().sfx_block_error_curve(
        _ptr(calib), _DT[calib.dtype], S, K, _ptr(W), _DT[W.dtype], N,
        ctypes.cast(lv, ctypes.c_void_p), P, ctypes.cast(err, ctypes.c_void_p),
        ctypes.cast(thr, ctypes.c_void_p), _ptr(buf), buf.numel(), _stream(stream)))
    return [float(v) for v in err], [float(v) for v in thr]


def sfx_greedy_allocate(err, weights, step, target):
    """Per-block levels from the greedy rounds (host only). err: [M][P] nested lists."""
    M, P = len(err), len(err[0])
    e = (ctypes.c_double * (M * P))(*[float(v) for row in err for v in row])
    w = (ctypes.c_double * M)(*[float(v) for v in weights])
    out = (ctypes.c_int * M)()
    _check("sfx_greedy_allocate", load().sfx_greedy_allocate(
        ctypes.cast(e, ctypes.c_void_p), ctypes.cast(w, ctypes.c_void_p), M, P, float(step),
        float(target), ctypes.cast(out, ctypes.c_void_p)))
    return [int(v) for v in out]


def sfx_device_sm_count() -> int:
    return int(load().sfx_device_sm_count())


GEMV_KERNELS = ("cuda_cores", "union_tcgen05", "union_mma")

SFX_PLAN_UNION_KERNEL, SFX_PLAN_UNION_MIN_B, SFX_PLAN_GEMV_NT, SFX_PLAN_GEMV_S, SFX_PLAN_UNION_S, \
    SFX_PLAN_MMA_CHUNKS, SFX_PLAN_DENSE, SFX_PLAN_TEST_STALL, SFX_PLAN_MOE_CHUNK = range(9)
DENSE_UNION_ONLY, DENSE_ONLY, DENSE_ONLY_TCGEN05 = 1, 2, 3
UNION_TCGEN05, UNION_MMA = 1, 2


def sfx_set_plan_override(key: int, value: int):
    """Override one launch-plan knob (0 = the planner's choice); tuning and tests only."""
    _check("sfx_set_plan_override", load().sfx_set_plan_override(int(key), int(value)))


def sfx_set_wait_limit_ns(ns: int):
    """Limit of the kernels' bounded waits in ns (0: the 2 s default)."""
    _check("sfx_set_wait_limit_ns", load().sfx_set_wait_limit_ns(int(ns)))


class plan_overrides:
    """Context manager: set plan overrides {key: value} and restore the planner on exit."""

    def __init__(self, **kv):
        names = {"union_kernel": SFX_PLAN_UNION_KERNEL, "union_min_b": SFX_PLAN_UNION_MIN_B,
                 "gemv_nt": SFX_PLAN_GEMV_NT, "gemv_s": SFX_PLAN_GEMV_S,
                 "union_s": SFX_PLAN_UNION_S, "mma_chunks": SFX_PLAN_MMA_CHUNKS,
                 "dense": SFX_PLAN_DENSE, "test_stall": SFX_PLAN_TEST_STALL,
                 "moe_chunk": SFX_PLAN_MOE_CHUNK}
        self.kv = {names[k]: v for k, v in kv.items()}

    def __enter__(self):
        for k, v in self.kv.items():
            sfx_set_plan_override(k, v)
        return self

    def __exit__(self, *exc):
        for k in self.kv:
            sfx_set_plan_override(k, 0)


def sfx_gemv_plan(B, K, N, flags=0, idx_mode=False) -> dict:
    """The launch plan sfx_sparse_gemv takes for these sizes (host only)."""
    out = (ctypes.c_int * 6)()
    _check("sfx_gemv_plan", load().sfx_gemv_plan(int(B), int(K), int(N), int(flags),
                                                  1 if idx_mode else 0,
                                                  ctypes.cast(out, ctypes.c_void_p)))
    return {"kernel": GEMV_KERNELS[out[0]], "NT": out[1], "S": out[2], "col_tiles": out[3],
            "chunks": out[4], "slice": out[5]}
