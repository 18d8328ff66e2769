"""Host-side checks of libawq that need no GPU: the library loads, exports every entry point that
include/awq.h declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

from weight_only_quantization_act_b200 import awq, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "awq.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return awq.load_library()


def declared_functions():
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(awq_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("awq_act_stats", "awq_search", "awq_quantize_pack", "awq_search_workspace_size",
                     "awq_last_error"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", awq.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(\w+)$", out, flags=re.M))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert hasattr(lib, n)
    assert set(awq.SIGNATURES) == set(declared_functions())
    # nothing else leaks out of the library (hidden visibility)
    assert all(e.startswith("awq_") for e in exported if not e.startswith("_")), sorted(exported)[:20]


def test_version_and_sizes(lib):
    assert lib.awq_version() == 100
    assert lib.awq_search_workspace_size(512, 256, 256, 128, 20) > 20 * 256 * 256 * 2
    assert lib.awq_search_workspace_size(512, 256, 256, 64, 20) == 0
    assert lib.awq_act_stats_workspace_size(512, 256) >= 2 * 256 * 8
    assert lib.awq_scale_table_workspace_size(256, 65) == 0


def test_layout_geometry(lib):
    lay = awq.search_layout(300, 384, 600, 20)
    assert (lay.tile_n, lay.tile_o) == (256, 256)
    assert (lay.tiles_n, lay.tiles_o) == (2, 3)
    assert lay.partials_per_tile == 8
    assert lay.partials_offset % 8 == 0
    assert lay.workspace_bytes == awq.search_workspace_size(300, 384, 600, 20)


FAKE = ctypes.c_void_p(1 << 20)        # never dereferenced: every call below fails validation first
MISALIGNED = ctypes.c_void_p((1 << 20) + 4)


def status_and_message(lib, rc):
    return rc, lib.awq_last_error().decode()


def test_search_rejects_bad_arguments(lib):
    ws = 1 << 30
    common = dict(N=512, K=256, ldx=256, O=256, ldw=256)

    def call(X=FAKE, N=512, K=256, ldx=256, W=FAKE, O=256, ldw=256, act=FAKE, group=128, n_grid=20, flags=0,
             wsp=FAKE, wsb=ws, losses=FAKE, best=FAKE, scales=FAKE):
        return lib.awq_search_ex(X, N, K, ldx, W, O, ldw, act, group, n_grid, flags, wsp, wsb, losses, best,
                                 scales, None)

    assert call(group=64) == 2
    assert call(n_grid=0) == 1 and call(n_grid=65) == 1
    assert call(X=None) == 1
    assert call(X=MISALIGNED) == 1
    assert call(K=200, ldx=200, ldw=200) == 1            # not a multiple of 128
    assert call(ldx=100) == 1                            # stride below K
    assert call(ldx=260) == 1                            # stride not a multiple of 8
    assert call(N=0) == 1 and call(O=0) == 1
    assert call(act=None) == 1 and call(scales=None) == 1
    assert call(flags=0x8) == 1
    assert call(wsp=None) == 3
    assert call(wsb=1000) == 3
    rc, msg = status_and_message(lib, call(wsb=1000))
    assert rc == 3 and "workspace" in msg
    assert common


def test_other_entry_points_reject_bad_arguments(lib):
    assert lib.awq_act_stats(None, 10, 256, 256, FAKE, 1 << 20, FAKE, None) == 1
    assert lib.awq_act_stats(FAKE, 10, 255, 256, FAKE, 1 << 20, FAKE, None) == 1
    assert lib.awq_act_stats(FAKE, 10, 256, 256, FAKE, 8, FAKE, None) == 3
    assert lib.awq_act_stats(FAKE, 0, 256, 256, FAKE, 1 << 20, FAKE, None) == 1
    # more than 65535 chunks of 256 rows (the chunk-sum grid's y extent): rejected before any launch
    rows = 65535 * 256 + 1
    assert lib.awq_act_stats(FAKE, rows, 2, 8, FAKE, 1 << 30, FAKE, None) == 1
    assert "65535 chunks" in lib.awq_last_error().decode()
    assert lib.awq_act_stats_noalloc(FAKE, rows, 2, 8, FAKE, None) == 1
    assert "65535 chunks" in lib.awq_last_error().decode()
    assert lib.awq_search_ex(FAKE, 512, 256, 256, FAKE, rows, 256, FAKE, 128, 20, 0x10, FAKE, 1 << 40, FAKE, FAKE,
                             FAKE, None) == 1
    assert "65535 chunks" in lib.awq_last_error().decode()
    assert lib.awq_quantize_pack(FAKE, 4, 256, 256, FAKE, 32, FAKE, FAKE, FAKE, None) == 2
    assert lib.awq_quantize_pack(FAKE, 4, 192, 192, FAKE, 128, FAKE, FAKE, FAKE, None) == 1
    assert lib.awq_quantize_pack(FAKE, 4, 256, 256, None, 128, FAKE, FAKE, FAKE, None) == 1
    assert lib.awq_quantize_pack_ex(FAKE, 4, 256, 256, FAKE, 128, 0x2, FAKE, FAKE, FAKE, None) == 1
    assert lib.awq_scale_table(FAKE, 256, 0, 0, FAKE, 1 << 20, FAKE, None) == 1
    assert lib.awq_scale_table(FAKE, 256, 20, 0x1, FAKE, 1 << 20, FAKE, None) == 1
    assert lib.awq_scale_table(FAKE, 256, 20, 0, FAKE, 4, FAKE, None) == 3
    assert lib.awq_search_status(None, 0, None) == 3
    assert lib.awq_search_get_layout(10, 256, 10, 128, 20, None) == 1


def test_binding_fails_loudly_without_library(tmp_path):
    saved = awq._lib
    try:
        awq._lib = None
        with pytest.raises(RuntimeError, match="libawq.so not found"):
            awq.load_library(str(tmp_path / "missing.so"))
    finally:
        awq._lib = saved


def test_next_row_entry_points_reject_bad_arguments(lib):
    bad8 = ctypes.c_void_p((1 << 20) + 4)  # 4-byte aligned only
    # INT8 pack: W, K % 8, null outputs, codes alignment, flags
    assert lib.awq_quantize_pack_int8(None, 4, 256, 256, FAKE, 0, FAKE, FAKE, None) == 1
    assert lib.awq_quantize_pack_int8(FAKE, 4, 252, 256, FAKE, 0, FAKE, FAKE, None) == 1
    assert lib.awq_quantize_pack_int8(FAKE, 4, 256, 256, None, 0, FAKE, FAKE, None) == 1
    assert lib.awq_quantize_pack_int8(FAKE, 4, 256, 256, FAKE, 0, bad8, FAKE, None) == 1
    assert lib.awq_quantize_pack_int8(FAKE, 4, 256, 256, FAKE, 0x40, FAKE, FAKE, None) == 1
    # scale folding: operands, C % 8, s, op, in place with different strides
    for fn in (lib.awq_scale_columns, lib.awq_scale_rows):
        assert fn(None, 4, 256, 256, FAKE, 0, FAKE, 256, None) == 1
        assert fn(FAKE, 4, 252, 256, FAKE, 0, FAKE, 256, None) == 1
        assert fn(FAKE, 4, 256, 256, None, 0, FAKE, 256, None) == 1
        assert fn(FAKE, 4, 256, 256, FAKE, 2, FAKE, 256, None) == 1
        assert fn(FAKE, 4, 256, 256, FAKE, 1, FAKE, 264, None) == 1
    # W4A16: shapes, codes, workspace
    ws = lib.awq_w4a16_workspace_size(256, 256)
    assert ws > 256 * 1024 and lib.awq_w4a16_workspace_size(64, 256) == 0

    def w4(X=FAKE, M=16, K=256, ldx=256, codes=FAKE, steps=FAKE, zeros=FAKE, O=256, Y=FAKE, ldy=256, wsp=FAKE,
           wsb=ws):
        return lib.awq_w4a16_gemm(X, M, K, ldx, codes, steps, zeros, O, Y, ldy, wsp, wsb, None)

    assert w4(X=None) == 1 and w4(Y=None) == 1
    assert w4(M=0) == 1
    assert w4(K=192, ldx=192) == 1          # K % 128
    assert w4(O=252, ldy=256) == 1          # O % 8
    assert w4(codes=None) == 1 and w4(codes=bad8) == 1 and w4(zeros=None) == 1
    assert w4(wsp=None) == 3 and w4(wsb=ws - 1) == 3
    rc, msg = status_and_message(lib, w4(wsb=16))
    assert rc == 3 and "workspace" in msg
    assert w4(wsp=bad8) == 1
    # the allocation-free statistic: operands, and a shape beyond its fixed scratch array
    assert lib.awq_act_stats_noalloc(None, 16, 256, 256, FAKE, None) == 1
    assert lib.awq_act_stats_noalloc(FAKE, 16, 256, 256, None, None) == 1
    assert lib.awq_act_stats_noalloc(FAKE, 1 << 20, 1 << 20, 1 << 20, FAKE, None) == 1


def test_w4a16_workspace_covers_its_regions(lib):
    # header (512 B) + the fixed few-token counter region (65536 x 4 B) + group-major steps and zeros
    # (K/128 x O rounded up to 256, fp32, each) + the few-token X' copy and group sums + split-K partials
    fixed = 512 + 65536 * 4
    for K, O in [(128, 8), (256, 256), (4096, 4096), (14336, 4096), (28672, 8192), (4096, 28672)]:
        ws = lib.awq_w4a16_workspace_size(K, O)
        o_pad = (O + 255) // 256 * 256
        assert ws >= fixed + 2 * (K // 128) * o_pad * 4, (K, O, ws)
        assert ws % 256 == 0
    assert lib.awq_w4a16_workspace_size(127, 8) == 0 and lib.awq_w4a16_workspace_size(128, 0) == 0
