"""Launch plans of the sparse GEMV (host logic, no GPU).

sfx_gemv_plan reports the kernel family, tile and K splits that sfx_sparse_gemv
launches. The values pinned here are the choices measured on B200 (148 SMs);
the invariants hold for any device.
"""
import pytest

from sparse_input_gemv_b200 import binding as sb

SHAPES = {  # (K, N) of the Llama-3 8B / 70B projections and the Phi-2 down projection
    "qkv": (4096, 6144), "o": (4096, 4096), "8b_gate_up": (4096, 28672),
    "8b_down": (14336, 4096), "70b_gate_up": (8192, 57344), "70b_down": (28672, 8192),
    "phi2_down": (10240, 2560), "ragged": (1000, 264),
}


@pytest.fixture(autouse=True)
def _lib():
    sb.load()
    for k in range(9):
        sb.sfx_set_plan_override(k, 0)


@pytest.mark.parametrize("name", list(SHAPES))
@pytest.mark.parametrize("B", [1, 2, 3, 4, 8, 16])
def test_plan_invariants(name, B):
    K, N = SHAPES[name]
    p = sb.sfx_gemv_plan(B, K, N)
    # the batch-union kernel from 3 tokens on, CUDA cores below
    assert p["kernel"] == ("union_mma" if B >= 3 else "cuda_cores")
    # the column tiles cover N exactly once
    assert (p["col_tiles"] - 1) * p["NT"] < N <= p["col_tiles"] * p["NT"]
    # the K splits cover K: S slices of `slice` rows, the last one non-empty
    assert (p["S"] - 1) * p["slice"] < K <= p["S"] * p["slice"]
    if p["kernel"] == "union_mma":
        assert p["chunks"] in (1, 2, 4, 8) and p["NT"] == 64 * p["chunks"]
        assert p["slice"] % 256 == 0 and p["slice"] <= 16384
    else:
        assert p["chunks"] == 0 and p["NT"] in (256, 512, 1024, 2048)
        assert p["slice"] % 32 == 0


def test_plan_pins_measured_choices():
    if sb.sfx_device_sm_count() != 148:
        pytest.skip("pinned for a 148-SM B200")
    pin = lambda B, name: {k: sb.sfx_gemv_plan(B, *SHAPES[name])[k] for k in ("NT", "S", "chunks")}
    # batch 1, CUDA cores: 256-column tiles for N = 4096 / 6144, 512 for 28672,
    # K splits filling one wave of 296 resident CTAs
    assert pin(1, "qkv") == {"NT": 256, "S": 12, "chunks": 0}
    assert pin(1, "o") == {"NT": 256, "S": 16, "chunks": 0}
    assert pin(1, "8b_gate_up") == {"NT": 512, "S": 5, "chunks": 0}
    assert pin(1, "8b_down") == {"NT": 256, "S": 18, "chunks": 0}
    # 16 tokens, mma.sync union: fewest K splits; among those the widest tile
    # with at least 1.5 CTAs per SM (222 at 148 SMs)
    assert pin(16, "8b_gate_up") == {"NT": 128, "S": 1, "chunks": 2}
    assert pin(16, "70b_gate_up") == {"NT": 256, "S": 1, "chunks": 4}
    assert pin(16, "70b_down") == {"NT": 64, "S": 2, "chunks": 1}
    assert pin(16, "8b_down") == {"NT": 64, "S": 4, "chunks": 1}
    assert pin(16, "qkv") == {"NT": 64, "S": 3, "chunks": 1}


def test_plan_one_wave_at_batch_one():
    # 1- and 2-slot CUDA-core kernels run two CTAs per SM: the grid fits one wave
    slots = 2 * sb.sfx_device_sm_count()
    for K, N in SHAPES.values():
        for B in (1, 2):
            p = sb.sfx_gemv_plan(B, K, N)
            assert p["col_tiles"] * p["S"] <= slots, (K, N, B, p)


def test_plan_flags_and_overrides():
    K, N = SHAPES["8b_gate_up"]
    # SFX_FLAG_CUDA_CORES keeps a batch on CUDA cores; an index list is batch 1 only
    assert sb.sfx_gemv_plan(16, K, N, flags=sb.SFX_FLAG_CUDA_CORES)["kernel"] == "cuda_cores"
    assert sb.sfx_gemv_plan(1, K, N, idx_mode=True)["kernel"] == "cuda_cores"
    with pytest.raises(sb.SfxError):
        sb.sfx_gemv_plan(2, K, N, idx_mode=True)
    with pytest.raises(sb.SfxError):
        sb.sfx_gemv_plan(17, K, N)
    # the tcgen05 union kernel: 128-column tiles, from 5 tokens on
    with sb.plan_overrides(union_kernel=sb.UNION_TCGEN05):
        assert sb.sfx_gemv_plan(4, K, N)["kernel"] == "cuda_cores"
        p = sb.sfx_gemv_plan(5, K, N)
        assert p["kernel"] == "union_tcgen05" and p["NT"] == 128 and p["chunks"] == 0
    with sb.plan_overrides(union_kernel=sb.UNION_MMA, mma_chunks=8):
        assert sb.sfx_gemv_plan(16, K, N)["NT"] == 512
        with sb.plan_overrides(union_min_b=2):
            assert sb.sfx_gemv_plan(2, K, N)["kernel"] == "union_mma"
    # back to the planner once the overrides are released
    assert sb.sfx_gemv_plan(16, K, N)["NT"] == 128


def test_plan_overrides_reject_out_of_range_values():
    for key, bad in ((sb.SFX_PLAN_UNION_KERNEL, 3), (sb.SFX_PLAN_UNION_MIN_B, 1),
                     (sb.SFX_PLAN_UNION_MIN_B, 17), (sb.SFX_PLAN_GEMV_NT, 384),
                     (sb.SFX_PLAN_GEMV_S, -1), (sb.SFX_PLAN_MMA_CHUNKS, 3), (sb.SFX_PLAN_DENSE, 4),
                     (sb.SFX_PLAN_TEST_STALL, 2), (sb.SFX_PLAN_MOE_CHUNK, 15),
                     (sb.SFX_PLAN_MOE_CHUNK, 65), (9, 1), (-1, 0)):
        with pytest.raises(sb.SfxError):
            sb.sfx_set_plan_override(key, bad)
    # the library reads no environment variable for its plans
    import os
    os.environ["SFX_MMA_CHUNKS"] = "8"
    try:
        assert sb.sfx_gemv_plan(16, *SHAPES["8b_gate_up"])["NT"] == 128
    finally:
        del os.environ["SFX_MMA_CHUNKS"]


def test_workspace_covers_the_plan():
    # the workspace holds the split-K partials of the plan (S x B x N fp32) and the header
    for K, N in SHAPES.values():
        for B in (1, 4, 16):
            p = sb.sfx_gemv_plan(B, K, N)
            need = sb.sfx_workspace_bytes(sb.SFX_OP_SPARSE_GEMV, B, K, N, sb.SFX_BF16)
            parts = (p["S"] * B * N * 4) if p["S"] > 1 else 0
            assert need >= 256 + parts, (K, N, B, p, need)
