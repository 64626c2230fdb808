"""Host-side checks of the C ABI: the library loads, exports every entry point
that include/sa.h declares, and rejects bad arguments before any launch."""
import ctypes
import os
import subprocess

import pytest

import block_sparse_attention_softmax_b200 as sa
from block_sparse_attention_softmax_b200 import build as sa_build


@pytest.fixture(scope="module")
def lib():
    sa_build.build()
    return sa.load()


def test_library_exports_every_declared_symbol(lib):
    declared = sa.header_symbols()
    assert len(declared) >= 14
    out = subprocess.run(["nm", "-D", "--defined-only", sa.lib_path()], capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [s for s in declared if s not in exported]
    assert not missing, missing
    for s in declared:
        assert hasattr(lib, s)


def test_status_strings_and_version(lib):
    assert sa.sa_version() == 100
    names = {0: "SA_OK", -1: "SA_ERR_INVALID_ARG", -2: "SA_ERR_UNSUPPORTED", -3: "SA_ERR_ALIGN",
             -4: "SA_ERR_CUDA", -5: "SA_ERR_DEVICE_TIMEOUT", -6: "SA_ERR_WORKSPACE"}
    for code, name in names.items():
        assert sa.sa_status_string(code) == name
    assert sa.sa_status_string(42) == "SA_ERR_UNKNOWN"


P = ctypes.c_void_p


def test_argument_validation_without_launch(lib):
    fake = P(0x1000)          # never dereferenced: validation fails first
    # unsupported head dim / block sizes
    assert lib.sa_pool_blocks(fake, fake, 1, 1, 128, 96, 64, 64, fake, fake, None) == -2
    assert lib.sa_pool_blocks(fake, fake, 1, 1, 128, 64, 32, 64, fake, fake, None) == -2
    assert lib.sa_pool_blocks(fake, fake, 1, 1, 128, 64, 64, 128, fake, fake, None) == -2
    assert b"head dim" in lib.sa_last_error() or b"block" in lib.sa_last_error()
    # non-positive sizes and null pointers
    assert lib.sa_pool_blocks(fake, fake, 0, 1, 128, 64, 64, 64, fake, fake, None) == -1
    assert lib.sa_pool_blocks(None, fake, 1, 1, 128, 64, 64, 64, fake, fake, None) == -1
    # misaligned pointer
    assert lib.sa_pool_blocks(P(0x1004), fake, 1, 1, 128, 64, 64, 64, fake, fake, None) == -3
    # size limits of the header: B*H <= 65535, B*H*N*d < 2^40, n_kb <= 16384 for the mask
    assert lib.sa_pool_blocks(fake, fake, 2, 32768, 128, 64, 64, 64, fake, fake, None) == -2
    assert lib.sa_pool_blocks(fake, fake, 1, 65535, 200000, 128, 64, 64, fake, fake, None) == -2
    assert lib.sa_build_mask_workspace_size(1, 1, 16384 * 64 + 1, 64, 64, 64) > 0
    assert lib.sa_build_mask(fake, fake, 1, 1, 16384 * 64 + 1, 64, 64, 64, 0.1, 0.9, 0.0,
                             fake, fake, None, None, None, fake, 1 << 40, None) == -2
    assert b"16384" in lib.sa_last_error()
    # Top-k / Top-p ranges
    ws = lib.sa_build_mask_workspace_size(1, 1, 128, 64, 64, 64)
    assert ws > 0
    args = [fake, fake, 1, 1, 128, 64, 64, 64]
    assert lib.sa_build_mask(*args, 0.0, 0.9, 0.0, fake, fake, None, None, None, fake, ws, None) == -1
    assert lib.sa_build_mask(*args, 0.1, 1.5, 0.0, fake, fake, None, None, None, fake, ws, None) == -1
    assert lib.sa_build_mask(*args, 0.1, 0.9, float("nan"), fake, fake, None, None, None, fake, ws, None) == -1
    # workspace too small
    assert lib.sa_build_mask(*args, 0.1, 0.9, 0.0, fake, fake, None, None, None, fake, ws - 1, None) == -6
    # attention: exactly one mask form
    a = [fake, fake, fake, 1, 1, 128, 64, 64, 64]
    assert lib.sa_sparse_attn_fwd(*a, fake, fake, fake, 0.0, fake, None, None, 0, None) == -1
    assert lib.sa_sparse_attn_fwd(*a, None, None, None, 0.0, fake, None, None, 0, None) == -1
    assert lib.sa_sparse_attn_fwd(*a, fake, None, None, 0.0, fake, None, None, 0, None) == -1
    need = lib.sa_sparse_attn_workspace_size(1, 1, 128, 64, 64, 64, 1)
    assert need > 0 and lib.sa_sparse_attn_workspace_size(1, 1, 128, 64, 64, 64, 0) == 0
    assert lib.sa_sparse_attn_fwd(*a, None, None, fake, 0.0, fake, None, fake, need - 1, None) == -6
    # the blended form: o must not overlap o_l (size checks come first)
    blend = lambda o_l, o: lib.sa_sparse_attn_blend_fwd(*a, None, None, fake, 0.0, o_l, fake, o, None, fake, need,
                                                        None)
    assert blend(fake, fake) == -1
    assert blend(P(0x1000 + 128 * 64 * 2 - 16), fake) == -1
    assert b"overlap" in lib.sa_last_error()
    # linear branch and blend
    assert lib.sa_linear_branch(None, fake, fake, 1, 1, 128, 64, fake, fake, fake, fake, 1 << 20, None) == -1
    assert lib.sa_blend(fake, fake, fake, fake, None, 1, 1, 128, 64, fake, None, 0, None) == -1


def test_workspace_sizes_scale_with_shape(lib):
    small = lib.sa_build_mask_workspace_size(1, 2, 1024, 64, 64, 64)
    big = lib.sa_build_mask_workspace_size(1, 40, 75600, 128, 128, 64)
    assert big > small > 0
    # scores of every row plus the pooled means
    nqb, nkb = 591, 1182
    assert big >= 40 * nqb * ((nkb + 3) // 4 * 4) * 4 + 40 * (nqb + nkb) * 128 * 4
    assert lib.sa_build_mask_workspace_size(1, 1, 128, 96, 64, 64) == 0   # unsupported -> 0
    assert lib.sa_linear_workspace_size(1, 40, 75600, 128) > 0


def test_build_mask_launch_count(lib):
    """The mask builder reports the launches it makes for a shape: three for
    the score-matrix path (up to 32 MiB of fp32 scores), six for the candidate
    path, zero for a rejected shape; SA_MASK_BUILDER overrides the choice."""
    import os
    saved = os.environ.pop("SA_MASK_BUILDER", None)
    try:
        assert lib.sa_build_mask_launches(1, 12, 32760, 128, 128, 64) == 3     # 6.3 MB of scores
        assert lib.sa_build_mask_launches(1, 40, 75600, 128, 128, 64) == 6     # 112 MB of scores
        assert lib.sa_build_mask_launches(1, 40, 245760, 128, 128, 64) == 6
        assert lib.sa_build_mask_launches(1, 1, 128, 96, 64, 64) == 0          # unsupported d
        os.environ["SA_MASK_BUILDER"] = "candidates"
        assert lib.sa_build_mask_launches(1, 12, 32760, 128, 128, 64) == 6
        os.environ["SA_MASK_BUILDER"] = "matrix"
        assert lib.sa_build_mask_launches(1, 40, 75600, 128, 128, 64) == 3
    finally:
        os.environ.pop("SA_MASK_BUILDER", None)
        if saved is not None:
            os.environ["SA_MASK_BUILDER"] = saved


def test_diagnostic_entry_points_validate_before_launch(lib):
    fake = P(0x1000)
    assert lib.sa_diag_exp2(fake, fake, fake, -1, None) == -1
    assert lib.sa_diag_exp2(None, fake, fake, 8, None) == -1
    assert lib.sa_diag_exp2(None, None, None, 0, None) == 0      # nothing to do, nothing launched
    assert lib.sa_diag_wait_timeout(None, None) == -1


def test_permutation_entry_points_validate_before_launch(lib):
    fake = P(0x1000)
    tiles = (ctypes.c_int32 * 3)(1, 2, 0)
    assert lib.sa_tile_permutation(1, 4, 4, 4, ctypes.cast(tiles, P), fake, None) == -1   # tile dimension 0
    assert lib.sa_tile_permutation(0, 4, 4, 4, ctypes.cast(tiles, P), fake, None) == -1   # no heads
    assert lib.sa_tile_permutation(300, 4, 4, 4, ctypes.cast(tiles, P), fake, None) == -1
    assert lib.sa_permute_tokens(fake, fake, 1, 1, 64, 64, 0, fake, None) == -1           # y aliases x
    assert lib.sa_permute_tokens(fake, fake, 1, 1, 64, 96, 0, P(0x2000), None) == -2
    assert lib.sa_select_mask(fake, 1, 1, 4, 20000, 0.1, 0.9, fake, fake, None, None) == -2
    assert lib.sa_tile_heatmap(fake, fake, 1, 1, 128, 64, 64, 64, 0.0, fake, -1, fake, None, None) == -1


def test_low_bit_entry_points_validate_before_launch(lib):
    fake, other = P(0x1000), P(0x2000)
    # quantiser: shape, null and alignment checks
    assert lib.sa_quantize_fp8(fake, 1, 1, 64, 96, other, fake, None) == -2       # d unsupported
    assert lib.sa_quantize_fp8(fake, 0, 1, 64, 128, other, fake, None) == -1      # B < 1
    assert lib.sa_quantize_fp8(None, 1, 1, 64, 128, other, fake, None) == -1      # null input
    assert lib.sa_quantize_fp8(P(0x1001), 1, 1, 64, 128, other, fake, None) == -3  # misaligned
    # low-bit attention: d = 128 only, scales required, lists xor mask
    args = (fake, fake, fake, fake, fake, fake)
    assert lib.sa_sparse_attn_fp8_fwd(*args, 1, 1, 256, 64, 128, 64, fake, fake, None, 0.0, None, None,
                                      other, None, None, 0, None) == -2
    assert lib.sa_sparse_attn_fp8_fwd(fake, fake, fake, None, fake, fake, 1, 1, 256, 128, 128, 64, fake, fake,
                                      None, 0.0, None, None, other, None, None, 0, None) == -1
    assert lib.sa_sparse_attn_fp8_fwd(*args, 1, 1, 256, 128, 128, 64, None, None, None, 0.0, None, None,
                                      other, None, None, 0, None) == -1
    assert lib.sa_sparse_attn_fp8_fwd(*args, 1, 1, 256, 128, 128, 64, fake, fake, None, 0.0, fake, None,
                                      other, None, None, 0, None) == -1            # o_l without alpha
