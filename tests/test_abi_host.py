"""Host-side checks of the C ABI (no GPU work): the library loads, exports
every entry point include/vsa.h declares, and rejects bad arguments with the
documented status codes before touching the device."""
import ctypes
import os
import subprocess
import re

import pytest

from block_sparse_attention_30_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vsa.h")

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation returns first


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vsa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_expected_entry_points():
    names = declared_functions()
    for n in ["vsa_select_blocks", "vsa_sparse_attn_fwd", "vsa_linear_branch_fwd",
              "vsa_sparse_attn_fwd_train", "vsa_sparse_attn_bwd", "vsa_linear_branch_bwd",
              "vsa_gather_tiles", "vsa_scatter_tiles", "vsa_workspace_bytes",
              "vsa_device_status", "vsa_status_string", "vsa_quantize_qk_e4m3",
              "vsa_sparse_attn_fwd_e4m3", "vsa_sparse_linear_attn_fwd_e4m3"]:
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
        assert name in _lib.SIGNATURES, f"binding lacks {name}"


def test_status_strings(L):
    for code, name in _lib.STATUS_NAMES.items():
        assert L.vsa_status_string(code).decode() == name
    assert L.vsa_status_string(99).decode() == "VSA_ERR_UNKNOWN"


def test_num_tiles_and_workspace(L):
    assert L.vsa_num_tiles(21, 45, 80, 4, 4, 4) == 1440
    assert L.vsa_num_tiles(20, 28, 52, 4, 4, 4) == 455
    assert L.vsa_num_tiles(4, 32, 32, 4, 4, 4) == 64
    assert L.vsa_num_tiles(0, 4, 4, 4, 4, 4) == 0
    nt, B, h, d = 455, 1, 40, 128
    # status block + the selection's scratch: 256 bytes of counters, the
    # pooled means as fp32 hi + lo for q and k, the feature-major copy of the
    # k means (nt rounded up to 4), one fallback row of nt 64-bit keys for
    # each of at most 1024 CTAs (no nt^2 term)
    ntp = (nt + 3) // 4 * 4
    want = 256 + 256 + 4 * B * h * nt * d * 4 + B * h * d * ntp * 4 + 1024 * nt * 8
    assert L.vsa_workspace_bytes(B, h, d, 20, 28, 52, 4, 4, 4, 46) == want
    assert L.vsa_workspace_bytes(B, h, 96, 20, 28, 52, 4, 4, 4, 46) == 0       # d unsupported
    assert L.vsa_workspace_bytes(B, h, d, 20, 28, 52, 4, 4, 2, 46) == 0        # volume 32
    assert L.vsa_workspace_bytes(B, h, d, 20, 28, 52, 4, 4, 4, 0) == 0         # topk < 1
    assert L.vsa_workspace_bytes(B, h, d, 20, 28, 52, 4, 4, 4, 456) == 0       # topk > nt
    # tiny grids: the linear branch's backward scratch (two operand images of
    # 4*d*d + 4*d bytes per (b, head) and the fp32 (dS, dz) sums, the same
    # size, each third rounded up to 256 bytes) is larger than the selection
    # scratch and sets the size
    third = -(-2 * (4 * 128 * 128 + 4 * 128) // 256) * 256
    assert L.vsa_workspace_bytes(1, 2, 128, 4, 8, 8, 4, 4, 4, 2) == 256 + 3 * third


SHAPE = [1, 2, 128, 4, 8, 8, 4, 4, 4]       # nt = 4


def test_select_argument_validation(L):
    f = L.vsa_select_blocks
    big = 1 << 30
    assert f(FAKE, FAKE, *SHAPE, 0, FAKE, FAKE, big, None) == INVALID
    assert f(FAKE, FAKE, *SHAPE, 5, FAKE, FAKE, big, None) == INVALID
    assert f(None, FAKE, *SHAPE, 2, FAKE, FAKE, big, None) == INVALID
    assert f(FAKE + 8, FAKE, *SHAPE, 2, FAKE, FAKE, big, None) == INVALID      # misaligned q
    assert f(FAKE, FAKE, *SHAPE, 2, FAKE, None, big, None) == WORKSPACE
    assert f(FAKE, FAKE, *SHAPE, 2, FAKE, FAKE, 100, None) == WORKSPACE
    bad = list(SHAPE); bad[2] = 80
    assert f(FAKE, FAKE, *bad, 2, FAKE, FAKE, big, None) == UNSUPPORTED
    bad = list(SHAPE); bad[6] = 2
    assert f(FAKE, FAKE, *bad, 2, FAKE, FAKE, big, None) == UNSUPPORTED
    # 3300 cubes: 16 score rows of 3300 fp32 values no longer fit a CTA's
    # shared memory beside the rest of a work item's state
    wide = [1, 1, 128, 4, 4, 4 * 3300, 4, 4, 4]
    assert f(FAKE, FAKE, *wide, 2, FAKE, FAKE, big, None) == UNSUPPORTED
    assert L.vsa_select_blocks_noalloc(FAKE, FAKE, *wide, 2, FAKE, None) == UNSUPPORTED
    bad = list(SHAPE); bad[3] = 0
    assert f(FAKE, FAKE, *bad, 2, FAKE, FAKE, big, None) == INVALID


def test_fine_argument_validation(L):
    f = L.vsa_sparse_attn_fwd
    big = 1 << 20
    assert f(FAKE, FAKE, FAKE, FAKE, None, None, FAKE, *SHAPE, 0, FAKE, big, None) == INVALID
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, *SHAPE, 2, FAKE, big, None) == INVALID  # S w/o z
    assert f(FAKE, FAKE, FAKE, None, None, None, FAKE, *SHAPE, 2, FAKE, big, None) == INVALID
    assert f(FAKE, FAKE, FAKE, FAKE, None, None, FAKE + 2, *SHAPE, 2, FAKE, big, None) == INVALID
    assert f(FAKE, FAKE, FAKE, FAKE, None, None, FAKE, *SHAPE, 2, None, big, None) == WORKSPACE
    assert f(FAKE, FAKE, FAKE, FAKE, None, None, FAKE, *SHAPE, 2, FAKE, 64, None) == WORKSPACE
    bad = list(SHAPE); bad[2] = 256
    assert f(FAKE, FAKE, FAKE, FAKE, None, None, FAKE, *bad, 2, FAKE, big, None) == UNSUPPORTED
    # with the linear branch the workspace must hold the (S, z) operand image
    image = 2 * (4 * 128 * 128 + 4 * 128)
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, *SHAPE, 2, FAKE, 256 + image - 16, None) == WORKSPACE


def test_other_entry_points_validate(L):
    assert L.vsa_gather_tiles(None, FAKE, *SHAPE, None) == INVALID
    assert L.vsa_scatter_tiles(FAKE, FAKE + 4, *SHAPE, None) == INVALID
    assert L.vsa_linear_branch_fwd(FAKE, FAKE, None, FAKE, 1, 2, 128, 4, 8, 8, FAKE, 1024, None) == INVALID
    assert L.vsa_linear_branch_fwd(FAKE, FAKE, FAKE, FAKE, 1, 2, 32, 4, 8, 8, FAKE, 1024, None) == UNSUPPORTED
    assert L.vsa_linear_branch_fwd(FAKE, FAKE, FAKE, FAKE, 1, 2, 128, 4, 8, 8, None, 1024, None) == WORKSPACE
    lb = L.vsa_linear_branch_bwd
    third = -(-2 * (4 * 128 * 128 + 4 * 128) // 256) * 256
    ok_ws = 256 + 3 * third
    assert lb(*[FAKE] * 9, 0, 1, 2, 128, 4, 8, 8, FAKE, ok_ws - 16, None) == WORKSPACE
    assert lb(*[FAKE] * 9, 0, 1, 2, 128, 4, 8, 8, None, ok_ws, None) == WORKSPACE
    assert lb(FAKE, FAKE, FAKE, None, *[FAKE] * 5, 0, 1, 2, 128, 4, 8, 8, FAKE, ok_ws, None) == INVALID
    assert lb(*[FAKE] * 8, FAKE + 8, 0, 1, 2, 128, 4, 8, 8, FAKE, ok_ws, None) == INVALID   # misaligned dv
    assert lb(*[FAKE] * 9, 0, 1, 2, 96, 4, 8, 8, FAKE, ok_ws, None) == UNSUPPORTED
    assert lb(*[FAKE] * 9, 0, 0, 2, 128, 4, 8, 8, FAKE, ok_ws, None) == INVALID
    qz = L.vsa_quantize_qk_e4m3
    assert qz(*[FAKE] * 6, 1, 2, 96, 4, 8, 8, 4, 4, 4, None) == UNSUPPORTED
    assert qz(FAKE, FAKE, FAKE + 4, FAKE, FAKE, FAKE, 1, 2, 128, 4, 8, 8, 4, 4, 4, None) == INVALID
    fe = L.vsa_sparse_attn_fwd_e4m3
    assert fe(*[FAKE] * 7, 1, 2, 96, 4, 8, 8, 4, 4, 4, 2, FAKE, 1024, None) == UNSUPPORTED   # d = 96
    assert fe(*[FAKE] * 7, 1, 2, 128, 4, 8, 8, 4, 4, 4, 5, FAKE, 1024, None) == INVALID     # topk > nt
    assert fe(*[FAKE] * 6, FAKE + 2, 1, 2, 128, 4, 8, 8, 4, 4, 4, 2, FAKE, 1024, None) == INVALID
    assert fe(*[FAKE] * 7, 1, 2, 128, 4, 8, 8, 4, 4, 4, 2, FAKE, 8, None) == WORKSPACE
    fl = L.vsa_sparse_linear_attn_fwd_e4m3                 # q8 k8 sq sk q v idx S z out
    image = 2 * (4 * 128 * 128 + 4 * 128)
    assert fl(*[FAKE] * 10, 1, 2, 96, 4, 8, 8, 4, 4, 4, 2, FAKE, 1 << 20, None) == UNSUPPORTED   # d = 96
    assert fl(*[FAKE] * 10, 1, 2, 128, 4, 8, 8, 4, 4, 4, 0, FAKE, 1 << 20, None) == INVALID     # topk < 1
    assert fl(*[FAKE] * 7, None, FAKE, FAKE, 1, 2, 128, 4, 8, 8, 4, 4, 4, 2, FAKE, 1 << 20, None) == INVALID
    assert fl(*[FAKE] * 4, FAKE + 2, *[FAKE] * 5, 1, 2, 128, 4, 8, 8, 4, 4, 4, 2, FAKE, 1 << 20, None) == INVALID
    assert fl(*[FAKE] * 10, 1, 2, 128, 4, 8, 8, 4, 4, 4, 2, FAKE, 256 + image - 16, None) == WORKSPACE
    ft = L.vsa_sparse_attn_fwd_train
    assert ft(*[FAKE] * 7, *SHAPE, 2, None, 1 << 30, None) == WORKSPACE
    assert ft(*[FAKE] * 5, FAKE + 4, FAKE, *SHAPE, 2, FAKE, 1 << 30, None) == INVALID        # out_f32
    assert ft(*[FAKE] * 7, *SHAPE, 5, FAKE, 1 << 30, None) == INVALID                        # topk > nt
    bad = list(SHAPE); bad[2] = 96
    assert ft(*[FAKE] * 7, *bad, 2, FAKE, 1 << 30, None) == UNSUPPORTED
    bw = L.vsa_sparse_attn_bwd
    rows = 1 * 2 * 4                                       # B * heads * nt
    up = lambda x: -(-x // 256) * 256
    need = 256 + up(rows * 64 * 4) + up(1 * 2 * (4 + 1) * 4) + up(rows * 2 * 4)
    assert L.vsa_workspace_bytes(*SHAPE, 2) >= need
    assert bw(*[FAKE] * 10, *SHAPE, 2, FAKE, need - 16, None) == WORKSPACE
    assert bw(*[FAKE] * 7, FAKE + 8, FAKE, FAKE, *SHAPE, 2, FAKE, need, None) == INVALID      # dq
    assert bw(*[FAKE] * 10, *SHAPE, 0, FAKE, need, None) == INVALID                           # topk < 1
    # the transpose of the block index keeps one bitmap row of nt bits in
    # shared memory: 327680 cubes fit, 327681 do not (refused before any launch)
    edge = [1, 1, 128, 4, 4, 4 * 327680, 4, 4, 4]
    over = [1, 1, 128, 4, 4, 4 * 327681, 4, 4, 4]
    assert bw(*[FAKE] * 10, *edge, 2, FAKE, 16, None) == WORKSPACE                            # passes the limit
    assert bw(*[FAKE] * 10, *over, 2, FAKE, 1 << 40, None) == UNSUPPORTED
    assert L.vsa_workspace_init(None, 1024, None) == INVALID
    assert L.vsa_workspace_init(FAKE, 8, None) == WORKSPACE
    assert L.vsa_device_status(None, None) == INVALID
    assert L.vsa_selftest_wait_timeout(None, 1024, 1000, None) == WORKSPACE
    assert L.vsa_selftest_wait_timeout(FAKE, 1024, 0, None) == INVALID


def test_library_has_no_oracle_dependency():
    """The product library never links or exports the oracle: its dynamic
    dependencies (readelf's NEEDED entries) and its exported symbols (nm -D)
    name no oracle library or function, and no package source imports it."""
    dyn = subprocess.run(["readelf", "-d", _lib.LIB_PATH], capture_output=True, text=True, check=True).stdout
    needed = [ln for ln in dyn.splitlines() if "(NEEDED)" in ln]
    assert needed and not any("oracle" in ln for ln in needed), needed
    syms = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True,
                          check=True).stdout
    assert "vsa_select_blocks" in syms and "oracle" not in syms
    for root, _, files in os.walk(os.path.join(ROOT, "block_sparse_attention_30_b200")):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(root, fn), encoding="utf-8").read()
                assert "import oracle" not in src and "from oracle" not in src, fn


def test_cuda_failures_surface_as_status_codes(L):
    """Host-side error injection into the VSA_ERR_CUDA paths: on a machine
    without a CUDA device every CUDA runtime or driver call the library makes
    (launches, memsets, stream synchronisation, tensor-map encoding, symbol
    lookup) returns an error.  With arguments that pass validation, each entry
    point must report that as VSA_ERR_CUDA, never crash, never return OK."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("needs a machine without a CUDA device (fake pointers would reach a real launch)")
    CUDA = 4
    SH = (1, 2, 128, 4, 8, 8, 4, 4, 4)          # 4 cubes of 64 tokens, d = 128
    ws = L.vsa_workspace_bytes(*SH, 2)
    assert ws > 0
    assert L.vsa_workspace_init(FAKE, ws, None) == CUDA
    assert L.vsa_gather_tiles(FAKE, FAKE, *SH, None) == CUDA
    assert L.vsa_scatter_tiles(FAKE, FAKE, *SH, None) == CUDA
    assert L.vsa_select_blocks(FAKE, FAKE, *SH, 2, FAKE, FAKE, ws, None) == CUDA
    assert L.vsa_select_blocks_noalloc(FAKE, FAKE, *SH, 2, FAKE, None) == CUDA
    assert L.vsa_linear_branch_fwd(FAKE, FAKE, FAKE, FAKE, *SH[:6], FAKE, ws, None) == CUDA
    assert L.vsa_sparse_attn_fwd(*[FAKE] * 4, None, None, FAKE, *SH, 2, FAKE, ws, None) == CUDA
    assert L.vsa_sparse_attn_fwd(*[FAKE] * 7, *SH, 2, FAKE, ws, None) == CUDA          # with the linear branch
    assert L.vsa_sparse_attn_fwd_train(*[FAKE] * 7, *SH, 2, FAKE, ws, None) == CUDA
    assert L.vsa_sparse_attn_bwd(*[FAKE] * 10, *SH, 2, FAKE, ws, None) == CUDA
    assert L.vsa_linear_branch_bwd(*[FAKE] * 9, 0, *SH[:6], FAKE, ws, None) == CUDA
    assert L.vsa_quantize_qk_e4m3(*[FAKE] * 6, *SH, None) == CUDA
    assert L.vsa_sparse_attn_fwd_e4m3(*[FAKE] * 7, *SH, 2, FAKE, ws, None) == CUDA
    assert L.vsa_sparse_linear_attn_fwd_e4m3(*[FAKE] * 10, *SH, 2, FAKE, ws, None) == CUDA
    assert L.vsa_selftest_wait_timeout(FAKE, ws, 1000, None) == CUDA
    assert L.vsa_device_status(FAKE, None) == CUDA


def test_debug_check_build_exports_every_symbol():
    """The debug-check build (-DVSA_DEBUG_CHECKS: non-finite outputs and TMA
    boxes outside the grid are recorded in the status word) compiles for
    sm_100a and exports the same C ABI as the product library."""
    lib = build.build(debug_checks=True)
    assert lib.endswith("libvsa_debug.so") and os.path.exists(lib)
    syms = subprocess.run(["nm", "-D", "--defined-only", lib], capture_output=True, text=True, check=True).stdout
    for name in declared_functions():
        assert re.search(r"\b%s\b" % name, syms), name
