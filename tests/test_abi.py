"""The C-ABI library builds, loads and exports every symbol its header
declares; argument validation answers without touching the GPU.  CPU only:
no forward pass is run here."""
import re
import subprocess

import pytest

from structured_sub_quadratic_b200 import _build, api

HEADER = _build.os.path.join(_build.INCLUDE, "monarch_attn.h")


def declared_symbols():
    text = open(HEADER).read()
    return set(re.findall(r"^MONARCH_API\s+[\w\s\*]+?\b(monarch_attn_\w+)\s*\(", text, re.M))


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return api.load_library()


def test_header_and_binding_agree():
    syms = declared_symbols()
    assert len(syms) >= 10
    assert syms == set(api.SIGNATURES)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", _build.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT\s+(monarch_attn_\w+)$", out, re.M))
    assert declared_symbols() <= exported
    for name in declared_symbols():
        assert getattr(lib, name) is not None


def test_library_is_built_for_sm100a_only():
    """The build compiles every source for sm_100a and nothing else."""
    arch = _build.ARCH
    assert arch == ["-gencode", "arch=compute_100a,code=sm_100a"]
    flags = " ".join(_build.NVCC_FLAGS)
    assert "-arch" not in flags and "-gencode" not in flags


def test_version_and_strerror(lib):
    assert lib.monarch_attn_version() >= 1
    for st in (0, -1, -2, -3, -4, -5, 7):
        assert lib.monarch_attn_strerror(st)


@pytest.mark.parametrize("args,expect", [
    ((0, 1, 4, 4, 64, 1, 1, 1), api.MONARCH_ERR_INVALID_ARG),     # B < 1
    ((1, 1, 0, 4, 64, 1, 1, 1), api.MONARCH_ERR_INVALID_ARG),     # b1 < 1
    ((1, 1, 4, 4, 64, -1, 1, 1), api.MONARCH_ERR_INVALID_ARG),    # T < 0
    ((1, 1, 4, 4, 64, 1, 5, 1), api.MONARCH_ERR_INVALID_ARG),     # c1 > b1
    ((1, 1, 4, 4, 64, 1, 1, 0), api.MONARCH_ERR_INVALID_ARG),     # c2 < 1
    ((1, 1, 4, 4, 512, 1, 1, 1), api.MONARCH_ERR_UNSUPPORTED),    # d > 256
])
def test_invalid_arguments_are_rejected_before_any_launch(lib, args, expect):
    # valid-looking (aligned, non-null) fake pointers: validation fails first
    p = 1 << 20
    assert lib.monarch_attn_fwd(p, 2 * p, 3 * p, 4 * p, *args, None) == expect
    assert lib.monarch_attn_workspace_bytes(*args, 0) == 0


def test_null_misaligned_and_overlapping_pointers_are_rejected(lib):
    p = 1 << 20
    sizes = (1, 1, 4, 4, 64, 1, 1, 1)
    assert lib.monarch_attn_fwd(None, p, p, p, *sizes, None) == api.MONARCH_ERR_INVALID_ARG
    assert lib.monarch_attn_fwd(p + 2, 2 * p, 3 * p, 4 * p, *sizes, None) == \
        api.MONARCH_ERR_INVALID_ARG
    # out overlapping q (16*64*2 bytes of q starting at p)
    assert lib.monarch_attn_fwd(p, 2 * p, 3 * p, p + 256, *sizes, None) == \
        api.MONARCH_ERR_INVALID_ARG
    assert lib.monarch_attn_fwd_host(9, p, p, p, p, *sizes, None) == api.MONARCH_ERR_INVALID_ARG


def test_workspace_bytes_scale_with_shape(lib):
    w1 = lib.monarch_attn_workspace_bytes(1, 12, 90, 52, 128, 1, 1, 1, 0)
    w2 = lib.monarch_attn_workspace_bytes(2, 12, 90, 52, 128, 1, 1, 1, 0)
    w3 = lib.monarch_attn_workspace_bytes(1, 12, 90, 52, 128, 2, 1, 1, 0)
    assert 0 < w1 < w2 and w1 < w3


@pytest.mark.parametrize("dtype,f,h,w,layout,expect", [
    (api.DTYPE_BF16, 2, 3, 4, 6, api.MONARCH_ERR_INVALID_ARG),    # unknown layout
    (api.DTYPE_BF16, 2, 3, 4, -1, api.MONARCH_ERR_INVALID_ARG),   # unknown layout
    (7, 2, 3, 4, 1, api.MONARCH_ERR_INVALID_ARG),                 # unknown dtype
    (api.DTYPE_BF16, 0, 3, 4, 1, api.MONARCH_ERR_INVALID_ARG),    # empty latent
    (api.DTYPE_F32, 2, 3, 4, 1, api.MONARCH_ERR_INVALID_ARG),     # null pointers (after the shape)
])
def test_video_layout_entry_validates_before_any_launch(lib, dtype, f, h, w, layout, expect):
    st = lib.monarch_attn_fwd_video(dtype, None, None, None, None, 1, 1, f, h, w, layout, 64, 1,
                                    1, 1, None)
    assert st == expect


def test_video_blocks_of_each_layout():
    f, h, w = 3, 30, 52
    got = {name: api.video_blocks(f, h, w, name) for name in api.LAYOUTS}
    assert got == {"fh,w": (90, 52), "w,fh": (52, 90), "f,hw": (3, 1560), "hw,f": (1560, 3),
                   "fw,h": (156, 30), "h,fw": (30, 156)}


@pytest.mark.parametrize("d,T,expect", [
    (96, 1, api.MONARCH_ERR_UNSUPPORTED),     # d outside {64, 128}: checked before sizes
    (0, 1, api.MONARCH_ERR_UNSUPPORTED),
    (-5, 1, api.MONARCH_ERR_UNSUPPORTED),
    (256, 1, api.MONARCH_ERR_UNSUPPORTED),
    (64, -1, api.MONARCH_ERR_INVALID_ARG),
])
def test_noalloc_entry_validates_before_any_launch(lib, d, T, expect):
    p = 1 << 20
    assert lib.monarch_attn_fwd_noalloc(p, 2 * p, 3 * p, 4 * p, 1, 1, 4, 4, d, T, 1, 1,
                                        None) == expect
    assert lib.monarch_attn_fwd_noalloc(None, p, p, p, 1, 1, 4, 4, 64, 1, 1, 1, None) == \
        api.MONARCH_ERR_INVALID_ARG


@pytest.mark.parametrize("dtype,n_real,pad_front,expect", [
    (api.DTYPE_BF16, 0, 1, api.MONARCH_ERR_INVALID_ARG),     # no real token
    (api.DTYPE_BF16, 17, 1, api.MONARCH_ERR_INVALID_ARG),    # more than b1*b2 = 16
    (api.DTYPE_BF16, 10, 2, api.MONARCH_ERR_INVALID_ARG),    # pad_front not 0/1
    (5, 10, 1, api.MONARCH_ERR_INVALID_ARG),                 # unknown dtype
])
def test_padded_entry_validates_before_any_launch(lib, dtype, n_real, pad_front, expect):
    p = 1 << 20
    assert lib.monarch_attn_fwd_padded(dtype, p, 2 * p, 3 * p, 4 * p, 1, 1, n_real, 4, 4,
                                       pad_front, 64, 1, 1, 1, None) == expect


def test_backward_entry_validates_before_any_launch(lib):
    p = 1 << 20
    sizes = (1, 1, 4, 4, 64)
    # T other than 1
    assert lib.monarch_attn_bwd(0, p, 2 * p, 3 * p, 4 * p, 5 * p, 6 * p, 7 * p, *sizes, 2, 1, 1,
                                None) == api.MONARCH_ERR_UNSUPPORTED
    # dq overlapping q, and dk overlapping dv
    assert lib.monarch_attn_bwd(0, p, 2 * p, 3 * p, 4 * p, p + 256, 6 * p, 7 * p, *sizes, 1, 1,
                                1, None) == api.MONARCH_ERR_INVALID_ARG
    assert lib.monarch_attn_bwd(0, p, 2 * p, 3 * p, 4 * p, 5 * p, 6 * p, 6 * p + 16, *sizes, 1,
                                1, 1, None) == api.MONARCH_ERR_INVALID_ARG
    assert lib.monarch_attn_bwd(9, p, 2 * p, 3 * p, 4 * p, 5 * p, 6 * p, 7 * p, *sizes, 1, 1, 1,
                                None) == api.MONARCH_ERR_INVALID_ARG
