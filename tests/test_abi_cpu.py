"""The C-ABI library loads and exports every symbol include/sfx.h declares.

No compute call is made here (no GPU): only host-side functions -- status
strings, workspace sizing and argument validation that rejects a call before
any launch.
"""
import ctypes
import os
import re

import pytest

from sparse_input_gemv_b200 import binding as sb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(sb.LIB_PATH):
        from sparse_input_gemv_b200 import build
        build.build()
    return sb.load()


def header_functions():
    text = open(os.path.join(ROOT, "include", "sfx.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sfx_[a-z_]+)\s*\(", text)))


def test_header_declares_the_five_calls():
    names = header_functions()
    for fn in ("sfx_calibrate_thresholds", "sfx_mask_compact", "sfx_sparse_gemv",
               "sfx_sparse_ffn_swiglu", "sfx_moe_expert_sparse"):
        assert fn in names


def test_header_is_plain_c_and_links(lib, tmp_path):
    # the boundary needs no C++ or CUDA types: a C99 program compiles against the
    # header and links against the library with the system C compiler
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_sfx.c"
    src.write_text(
        '#include "sfx.h"\n'
        "int main(void) {\n"
        "  int plan[6];\n"
        "  if (sfx_gemv_plan(1, 4096, 4096, 0, 0, plan) != SFX_OK) return 1;\n"
        "  return sfx_workspace_bytes(SFX_OP_SPARSE_GEMV, 1, 4096, 4096, SFX_BF16, 0, 0) >= 256 ? 0 : 2;\n"
        "}\n")
    exe = tmp_path / "use_sfx"
    lib_dir = os.path.dirname(sb.LIB_PATH)
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                        "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                        "-L", lib_dir, "-lsfx", f"-Wl,-rpath,{lib_dir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True)
    assert run.returncode == 0, (run.returncode, run.stderr)


def test_library_exports_every_declared_symbol(lib):
    names = header_functions()
    assert len(names) >= 12
    for fn in names:
        assert hasattr(lib, fn), f"{fn} declared in include/sfx.h but not exported"
        assert fn in sb.EXPORTED, f"{fn} has no binding signature"


def test_status_strings(lib):
    for code in range(0, -8, -1):
        s = lib.sfx_status_string(code).decode()
        assert s and s != "unknown status"
    assert lib.sfx_status_string(-99).decode() == "unknown status"


def test_workspace_sizes(lib):
    assert sb.sfx_workspace_bytes(sb.SFX_OP_SPARSE_GEMV, 1, 4096, 14336 * 2, sb.SFX_BF16) >= 256
    assert sb.sfx_workspace_bytes(sb.SFX_OP_FFN_SWIGLU, 1, 4096, 14336, sb.SFX_BF16) >= 14336 * 4
    assert sb.sfx_workspace_bytes(sb.SFX_OP_CALIBRATE, 64, 4096, 4, sb.SFX_BF16) >= 32768 * 4
    assert sb.sfx_workspace_bytes(sb.SFX_OP_MASK_COMPACT, 1, 10240, sb.SFX_SEL_TOPK_GLASS) >= \
        10240 * 20
    assert sb.sfx_workspace_bytes(99, 1, 1, 1) == 0
    assert sb.sfx_workspace_bytes(sb.SFX_OP_SPARSE_GEMV, 0, 10, 8) == 0


def _gemv(lib, x=0x1000, W=0x2000, y=0x3000, B=1, K=64, N=64, wdt=sb.SFX_BF16, xdt=sb.SFX_BF16,
          ydt=sb.SFX_BF16, idx=None, cnt=None, flags=0, ws=0x4000, ws_bytes=1 << 20):
    # fake (never dereferenced) pointers: every case below is rejected on the host
    return lib.sfx_sparse_gemv(x, xdt, B, K, W, wdt, N, 0.5, idx, cnt, y, ydt, flags, None, ws,
                               ws_bytes, None)


def test_gemv_rejects_bad_arguments_before_launch(lib):
    assert _gemv(lib, x=None) == -1
    assert _gemv(lib, B=0) == -1
    assert _gemv(lib, B=17) == -1
    assert _gemv(lib, N=4) == -1
    assert _gemv(lib, idx=0x5000, cnt=None) == -1
    assert _gemv(lib, idx=0x5000, cnt=0x6000, B=2) == -1
    assert _gemv(lib, flags=sb.SFX_FLAG_GELU | sb.SFX_FLAG_GELU_TANH) == -1
    assert _gemv(lib, wdt=sb.SFX_F32) == -2
    assert _gemv(lib, xdt=sb.SFX_F16) == -2          # bf16 weights, f16 activations
    assert _gemv(lib, W=0x2008) == -3                # not 16-byte aligned
    assert _gemv(lib, N=68) == -3                    # N % 8 != 0
    assert _gemv(lib, ws=None) == -4
    assert _gemv(lib, ws_bytes=16) == -4


def _gemv_mask(lib, x=0x1000, W=0x2000, mask=0x5000, y=0x3000, B=1, K=64, N=64,
               wdt=sb.SFX_BF16, xdt=sb.SFX_BF16, ydt=sb.SFX_BF16, flags=0, ws=0x4000,
               ws_bytes=1 << 20):
    # fake (never dereferenced) pointers: every case below is rejected on the host
    return lib.sfx_sparse_gemv_mask(x, xdt, B, K, W, wdt, N, mask, y, ydt, flags, ws, ws_bytes,
                                    None)


def test_gemv_on_a_mask_rejects_bad_arguments_before_launch(lib):
    assert _gemv_mask(lib, mask=None) == -1
    assert _gemv_mask(lib, x=None) == -1
    assert _gemv_mask(lib, B=0) == -1
    assert _gemv_mask(lib, B=17) == -1
    assert _gemv_mask(lib, N=4) == -1
    assert _gemv_mask(lib, flags=sb.SFX_FLAG_SWIGLU | sb.SFX_FLAG_GELU) == -1
    assert _gemv_mask(lib, wdt=sb.SFX_F32) == -2
    assert _gemv_mask(lib, flags=sb.SFX_FLAG_SWIGLU) == -2   # SwiGLU writes fp32 h
    assert _gemv_mask(lib, W=0x2008) == -3                   # not 16-byte aligned
    assert _gemv_mask(lib, N=68) == -3
    assert _gemv_mask(lib, ws_bytes=16) == -4


def test_other_entry_points_reject_bad_arguments(lib):
    VP = ctypes.c_void_p
    # calibration: P out of range, NaN sparsity
    sp = (ctypes.c_double * 1)(float("nan"))
    out = (ctypes.c_float * 1)()
    assert lib.sfx_calibrate_thresholds(VP(0x1000), sb.SFX_BF16, 4, 8, ctypes.cast(sp, VP), 0,
                                        ctypes.cast(out, VP), VP(0x2000), 1 << 20, None) == -1
    assert lib.sfx_calibrate_thresholds(VP(0x1000), sb.SFX_BF16, 4, 8, ctypes.cast(sp, VP), 1,
                                        ctypes.cast(out, VP), VP(0x2000), 1 << 20, None) == -1
    # mask_compact: k > K, union requested for GxO top-k, missing count buffer
    assert lib.sfx_mask_compact(VP(0x1000), sb.SFX_F32, 1, 16, sb.SFX_SEL_TOPK_GXO, 0.0, 17,
                                VP(0x2000), None, 0.5, None, None, VP(0x3000), None, None,
                                VP(0x4000), 1 << 20, None) == -1
    assert lib.sfx_mask_compact(VP(0x1000), sb.SFX_F32, 1, 16, sb.SFX_SEL_TOPK_GXO, 0.0, 4,
                                VP(0x2000), None, 0.5, None, None, VP(0x3000), VP(0x5000),
                                VP(0x6000), VP(0x4000), 1 << 20, None) == -7
    assert lib.sfx_mask_compact(VP(0x1000), sb.SFX_F32, 1, 16, sb.SFX_SEL_THRESHOLD, 0.0, 0,
                                None, None, 0.5, None, None, None, None, None,
                                VP(0x4000), 1 << 20, None) == -1
    # corrected GxO: the same limits as GxO (k <= K, K <= 32768, no union list)
    assert lib.sfx_mask_compact(VP(0x1000), sb.SFX_F32, 1, 16, sb.SFX_SEL_TOPK_CGXO, 0.0, 17,
                                VP(0x2000), None, 0.5, None, None, VP(0x3000), None, None,
                                VP(0x4000), 1 << 20, None) == -1
    assert lib.sfx_mask_compact(VP(0x1000), sb.SFX_F32, 1, 40000, sb.SFX_SEL_TOPK_CGXO, 0.0, 4,
                                VP(0x2000), None, 0.5, None, None, VP(0x3000), None, None,
                                VP(0x4000), 1 << 20, None) == -7
    assert lib.sfx_mask_compact(VP(0x1000), sb.SFX_F32, 1, 16, 4, 0.0, 4,
                                VP(0x2000), None, 0.5, None, None, VP(0x3000), None, None,
                                VP(0x4000), 1 << 20, None) == -1
    # FFN: misaligned down weights
    assert lib.sfx_sparse_ffn_swiglu(VP(0x1000), sb.SFX_BF16, 1, 64, 128, VP(0x2000), VP(0x3004),
                                     0.1, 0.1, VP(0x4000), sb.SFX_BF16, None, None, None, 0,
                                     VP(0x5000), 1 << 24, None) == -3
    # MoE: top_k > E
    assert lib.sfx_moe_expert_sparse(VP(0x1000), sb.SFX_BF16, VP(0x2000), 1, 64, 4, 64, 5,
                                     VP(0x3000), VP(0x4000), VP(0x5000), VP(0x6000), None, None,
                                     None, 0, VP(0x7000), sb.SFX_BF16, None, None, 0, VP(0x8000),
                                     1 << 24, None) == -1
    # MoE: the batch's x (B * d elements) must fit the expert kernel's shared memory
    assert lib.sfx_moe_expert_sparse(VP(0x1000), sb.SFX_BF16, VP(0x2000), 16, 8192, 4, 64, 2,
                                     VP(0x3000), VP(0x4000), VP(0x5000), VP(0x6000), None, None,
                                     None, 0, VP(0x7000), sb.SFX_BF16, None, None, 0, VP(0x8000),
                                     1 << 30, None) == -1
    # static-mask FFN: too many tokens, misaligned weights, fp32 weights
    assert lib.sfx_static_ffn(VP(0x1000), sb.SFX_BF16, 17, 64, 32, VP(0x2000), None, VP(0x3000),
                              VP(0x4000), VP(0x5000), 0, VP(0x6000), sb.SFX_BF16, VP(0x7000),
                              1 << 20, None) == -1
    assert lib.sfx_static_ffn(VP(0x1000), sb.SFX_BF16, 1, 64, 32, VP(0x2008), None, VP(0x3000),
                              VP(0x4000), VP(0x5000), 0, VP(0x6000), sb.SFX_BF16, VP(0x7000),
                              1 << 20, None) == -3
    assert lib.sfx_static_ffn(VP(0x1000), sb.SFX_F32, 1, 64, 32, VP(0x2000), None, VP(0x3000),
                              VP(0x4000), VP(0x5000), 0, VP(0x6000), sb.SFX_BF16, VP(0x7000),
                              1 << 20, None) == -2
    # MoE: the shared expert's three matrices come together or not at all
    assert lib.sfx_moe_expert_sparse(VP(0x1000), sb.SFX_BF16, VP(0x2000), 1, 64, 4, 64, 2,
                                     VP(0x3000), VP(0x4000), VP(0x5000), VP(0x6000), VP(0x9000),
                                     None, VP(0xa000), 64, VP(0x7000), sb.SFX_BF16, None, None, 0,
                                     VP(0x8000), 1 << 24, None) == -1
