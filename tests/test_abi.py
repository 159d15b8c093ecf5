"""Host-only checks of the C ABI: the library builds for sm_100a, loads, and
exports every entry point include/ft.h declares; argument validation rejects
bad calls before anything touches the GPU (these calls never reach CUDA)."""
import ctypes
import os
import re

import pytest

from bit_quantized_lora_b200 import _lib
from bit_quantized_lora_b200._lib import FtFp4, FtLinear

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ft.h")

FT_OK, FT_ERR_INVALID_ARG, FT_ERR_SHAPE, FT_ERR_ALIGN = 0, 1, 2, 3
FT_ERR_WORKSPACE = 6


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ft_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    return _lib.load(build_if_missing=True)


def test_every_declared_symbol_is_exported_and_bound(L):
    names = declared_functions()
    assert len(names) >= 8
    for n in names:
        assert hasattr(L, n), n
        assert n in _lib.SIGNATURES, n
    assert set(_lib.SIGNATURES) == set(names)


def test_struct_layouts_match_c():
    # int64 x4, float (+4 pad), two 48-byte views, six pointers
    assert ctypes.sizeof(FtFp4) == 48
    assert ctypes.sizeof(FtLinear) == 32 + 8 + 2 * 48 + 6 * 8 + 8 + 2 * 8


def test_status_strings(L):
    assert L.ft_status_str(0) == b"FT_OK"
    assert L.ft_status_str(2) == b"FT_ERR_SHAPE"
    assert L.ft_status_str(99) == b"FT_ERR_UNKNOWN"


def test_workspace_sizes_are_deterministic_and_monotone(L):
    a = L.ft_workspace_bytes(4608, 3072, 3072, 32, 16)
    b = L.ft_workspace_bytes(4608, 3072, 3072, 32, 16)
    c = L.ft_workspace_bytes(9216, 3072, 3072, 32, 16)
    assert a == b and c > a > 0
    assert L.ft_workspace_bytes(-1, 1, 1, 0, 0) == 0
    assert L.ft_quantize_workspace_bytes() == 256


def _view(rows, cols, blk, p=0x1000):
    return FtFp4(p, p, p, rows, cols, blk)


def test_quantize_validation_happens_on_the_host(L):
    v = _view(32, 64, 0)
    x = 0x10000
    # null input
    assert L.ft_quantize(None, 32, 64, 64, 0, None, ctypes.byref(v), x, 256, None) == FT_ERR_INVALID_ARG
    # bad block enum
    assert L.ft_quantize(x, 32, 64, 64, 7, None, ctypes.byref(v), x, 256, None) == FT_ERR_INVALID_ARG
    # cols not a multiple of 16
    v2 = _view(32, 60, 0)
    assert L.ft_quantize(x, 32, 60, 64, 0, None, ctypes.byref(v2), x, 256, None) == FT_ERR_SHAPE
    # 16x16 needs rows % 16 == 0
    v3 = _view(30, 64, 1)
    assert L.ft_quantize(x, 30, 64, 64, 1, None, ctypes.byref(v3), x, 256, None) == FT_ERR_SHAPE
    # view shape must match
    assert L.ft_quantize(x, 16, 64, 64, 0, None, ctypes.byref(v), x, 256, None) == FT_ERR_SHAPE
    # misaligned input pointer / leading dimension
    assert L.ft_quantize(x + 2, 32, 64, 64, 0, None, ctypes.byref(v), x, 256, None) == FT_ERR_ALIGN
    assert L.ft_quantize(x, 32, 64, 68, 0, None, ctypes.byref(v), x, 256, None) == FT_ERR_ALIGN
    # amax to compute but no workspace
    assert L.ft_quantize(x, 32, 64, 64, 0, None, ctypes.byref(v), None, 0, None) == FT_ERR_WORKSPACE
    # empty input: nothing to do, no launch
    v0 = _view(0, 64, 0)
    assert L.ft_quantize(x, 0, 64, 64, 0, None, ctypes.byref(v0), x, 256, None) == FT_OK


def _linear(N=256, K=256, r_s=16, r_l=16):
    p = 0x100000
    wk = FtFp4(p, p, p, N, K, 1)
    wn = FtFp4(p, p, p, K, N, 1)
    return FtLinear(N, K, r_s, r_l, 1.0, wk, wn, p, p, p, p, p, p)


def test_linear_validation_happens_on_the_host(L):
    x = 0x200000
    ws = L.ft_workspace_bytes(128, 256, 256, 16, 16)
    ok = _linear()
    bad_n = _linear(N=320)
    assert L.ft_linear_fwd(ctypes.byref(bad_n), x, 128, None, x, 0, x, None, x, ws, None) == FT_ERR_SHAPE
    bad_r = _linear(r_s=8)
    assert L.ft_linear_fwd(ctypes.byref(bad_r), x, 128, None, x, 0, x, None, x, ws, None) == FT_ERR_SHAPE
    big_r = _linear(r_s=80, r_l=64)
    assert L.ft_linear_fwd(ctypes.byref(big_r), x, 128, None, x, 0, x, None, x, ws, None) == FT_ERR_SHAPE
    assert L.ft_linear_fwd(None, x, 128, None, x, 0, x, None, x, ws, None) == FT_ERR_INVALID_ARG
    assert L.ft_linear_fwd(ctypes.byref(ok), x, 128, None, x, 5, x, None, x, ws, None) == FT_ERR_INVALID_ARG
    assert L.ft_linear_fwd(ctypes.byref(ok), x, 128, None, x, 0, x, None, x, ws - 1, None) == FT_ERR_WORKSPACE
    assert L.ft_linear_fwd(ctypes.byref(ok), x + 8, 128, None, x, 0, x, None, x, ws, None) == FT_ERR_ALIGN
    # the epilogue's amax word must be 4-byte aligned
    assert L.ft_linear_fwd(ctypes.byref(ok), x, 128, None, x, 0, x, x + 2, x, ws, None) == FT_ERR_ALIGN
    # the transposed weight view must share the scale grid
    shared = _linear()
    shared.w_n.scales = 0x300000
    assert L.ft_linear_fwd(ctypes.byref(shared), x, 128, None, x, 0, x, None, x, ws, None) == FT_ERR_INVALID_ARG
    # the weight operand images are required and 16-byte aligned
    no_sf = _linear()
    no_sf.op_n = None
    assert L.ft_linear_fwd(ctypes.byref(no_sf), x, 128, None, x, 0, x, None, x, ws, None) == FT_ERR_INVALID_ARG
    odd_sf = _linear()
    odd_sf.op_k = 0x100008
    assert L.ft_linear_fwd(ctypes.byref(odd_sf), x, 128, None, x, 0, x, None, x, ws, None) == FT_ERR_ALIGN
    # M = 0: nothing to do
    assert L.ft_linear_fwd(ctypes.byref(ok), x, 0, None, x, 0, x, None, x, ws, None) == FT_OK
    assert L.ft_linear_bwd(ctypes.byref(bad_n), x, x, x, 128, None, x, 0, x, x, x, ws, None) == FT_ERR_SHAPE
    assert L.ft_linear_bwd(ctypes.byref(ok), x, x, x, 128, None, x, 9, x, x, x, ws, None) == FT_ERR_INVALID_ARG


def test_workspace_qact_offsets_lie_inside_the_workspace(L):
    for M, N, K, rs, rl in [(4608, 3072, 3072, 32, 16), (128, 256, 256, 16, 16), (37, 512, 256, 0, 0)]:
        c, s, g = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
        assert L.ft_workspace_qact(M, N, K, rs, rl, ctypes.byref(c), ctypes.byref(s), ctypes.byref(g)) == FT_OK
        total = L.ft_workspace_bytes(M, N, K, rs, rl)
        C = max(N, K)
        # codes, scales and the tensor scale do not overlap and fit the workspace
        spans = sorted([(c.value, M * C // 2), (s.value, M * C // 16), (g.value, 4)])
        for (a, n), (b, _) in zip(spans, spans[1:]):
            assert a + n <= b
        assert spans[-1][0] + spans[-1][1] <= total
        assert c.value % 16 == 0 and s.value % 16 == 0
    bad = ctypes.c_size_t()
    assert L.ft_workspace_qact(-1, 1, 1, 0, 0, ctypes.byref(bad), ctypes.byref(bad), ctypes.byref(bad)) == FT_ERR_INVALID_ARG
    assert L.ft_workspace_qact(1, 1, 1, 0, 0, None, ctypes.byref(bad), ctypes.byref(bad)) == FT_ERR_INVALID_ARG


def test_weight_operand_packing_validation(L):
    # one 288 x 128-byte block (codes + scales) per 256 x 256 tile of the weight
    assert L.ft_weight_operand_bytes(3072, 3072) == 12 * 12 * 288 * 128
    assert L.ft_weight_operand_bytes(3072, 3072) == 3072 * 3072 // 2 * 9 // 8
    assert L.ft_weight_operand_bytes(-1, 256) == 0
    g = 0x100000
    assert L.ft_pack_weight_operands(None, g, g, 256, 256, g, g, None) == FT_ERR_INVALID_ARG
    assert L.ft_pack_weight_operands(g, g, None, 256, 256, g, g, None) == FT_ERR_INVALID_ARG
    assert L.ft_pack_weight_operands(g, g, g, 320, 256, g, g, None) == FT_ERR_SHAPE
    assert L.ft_pack_weight_operands(g, g, g, 256, 256, g + 8, g, None) == FT_ERR_ALIGN
    assert L.ft_pack_weight_operands(g, g, g, 0, 256, g, g, None) == FT_OK


def test_cooperative_quantizer_switch_is_host_only(L):
    """The launch-mode switch touches no device: it answers FT_OK on a host
    without a GPU and accepts any int (nonzero = cooperative)."""
    try:
        for on in (1, 0, 7, 0):
            assert L.ft_set_cooperative_quantizer(on) == 0
    finally:
        L.ft_set_cooperative_quantizer(0)


def test_gemm_mode_switch_is_host_only(L):
    """The GEMM tiling switch touches no device: modes 0 (CTA pairs) and 1
    (one CTA per tile) answer FT_OK without a GPU; any other mode is
    rejected and leaves the setting alone."""
    try:
        for mode in (1, 0, 1):
            assert L.ft_set_gemm_mode(mode) == 0
        for bad in (2, -1, 7):
            assert L.ft_set_gemm_mode(bad) == FT_ERR_INVALID_ARG
    finally:
        L.ft_set_gemm_mode(0)


def test_header_is_plain_c_and_the_library_links_from_c(L, tmp_path):
    """include/ft.h compiles as strict C11 (no C++ or CUDA headers) and a C
    program links libft_b200.so and runs its host-only entry points."""
    import shutil
    import subprocess
    from bit_quantized_lora_b200 import _lib
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    lib = _lib.lib_path()
    exe = tmp_path / "c_client"
    cmd = [gcc, "-std=c11", "-Wall", "-Wextra", "-pedantic", "-Werror",
           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_client.c"),
           "-o", str(exe), "-L", os.path.dirname(lib), "-l:" + os.path.basename(lib),
           "-Wl,-rpath," + os.path.dirname(lib)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr


def test_recorded_traffic_follows_kernel_code_not_comments(tmp_path, monkeypatch):
    """bench.py reports a kernel's ncu DRAM traffic only while the recorded
    source hash matches: a comment edit keeps the figure, a code edit drops
    it (the counters were taken on other code)."""
    import importlib.util
    import shutil
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    csrc = tmp_path / "bit_quantized_lora_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in ("k_qres.cuh", "ft_ptx.cuh", "ft_nvfp4.cuh"):
        shutil.copy(os.path.join(ROOT, "bit_quantized_lora_b200", "csrc", f), csrc / f)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_sha("k_qres.cuh")
    src = (csrc / "k_qres.cuh").read_text()
    (csrc / "k_qres.cuh").write_text(src.replace("#pragma once", "// a new comment\n/* and another */\n#pragma once", 1))
    assert bench.kernel_source_sha("k_qres.cuh") == h0
    (csrc / "k_qres.cuh").write_text(src.replace("constexpr int MAX_FS = 8;", "constexpr int MAX_FS = 6;", 1))
    assert bench.kernel_source_sha("k_qres.cuh") != h0


def test_1x16_weight_views_and_packing_validation(L):
    """The granularity ablation's weights: both views 1x16 with their own
    scales (W_res along K, W_res^T along N); a mixed pair is refused."""
    x = 0x200000
    ws = L.ft_workspace_bytes(128, 256, 256, 16, 16)
    g1 = _linear()
    g1.w_k.blk = 0
    g1.w_n.blk = 0
    g1.w_n.scales = 0x300000  # its own scales
    # with M = 0 the call validates the views and returns, launching nothing
    assert L.ft_linear_fwd(ctypes.byref(g1), x, 0, None, x, 0, x, None, x, ws, None) == FT_OK
    mixed = _linear()
    mixed.w_k.blk = 0
    assert L.ft_linear_fwd(ctypes.byref(mixed), x, 128, None, x, 0, x, None, x, ws, None) == FT_ERR_SHAPE
    no_sc = _linear()
    no_sc.w_k.blk = 0
    no_sc.w_n.blk = 0
    no_sc.w_n.scales = None
    assert L.ft_linear_fwd(ctypes.byref(no_sc), x, 128, None, x, 0, x, None, x, ws, None) == FT_ERR_INVALID_ARG
    g = 0x100000
    assert L.ft_pack_weight_operands_1x16(g, None, g, g, 256, 256, g, g, None) == FT_ERR_INVALID_ARG
    assert L.ft_pack_weight_operands_1x16(g, g, g, None, 256, 256, g, g, None) == FT_ERR_INVALID_ARG
    assert L.ft_pack_weight_operands_1x16(g, g, g, g, 256, 320, g, g, None) == FT_ERR_SHAPE
    assert L.ft_pack_weight_operands_1x16(g, g, g, g, 256, 256, g, g + 8, None) == FT_ERR_ALIGN
    assert L.ft_pack_weight_operands_1x16(g, g, g, g, 0, 256, g, g, None) == FT_OK


def test_precision_field_is_validated_on_the_host(L):
    """The precision configuration of a layer (the FourTune page's Table 4):
    out-of-range values and a 16-bit GEMM without its bf16 weight image are
    refused before any launch, as is a misaligned image."""
    x = 0x200000
    ws = L.ft_workspace_bytes(128, 256, 256, 16, 16)
    for prec, wd_k, wd_n, want in [(4, 0, 0, FT_ERR_INVALID_ARG), (-1, 0, 0, FT_ERR_INVALID_ARG),
                                   (1, 0, 0, FT_ERR_INVALID_ARG), (2, x, 0, FT_ERR_INVALID_ARG),
                                   (3, x, 0, FT_ERR_INVALID_ARG), (1, x + 8, 0, FT_ERR_ALIGN),
                                   (2, 0, x + 4, FT_ERR_ALIGN)]:
        lin = _linear()
        lin.precision, lin.wd_k, lin.wd_n = prec, wd_k or None, wd_n or None
        assert L.ft_linear_fwd(ctypes.byref(lin), x, 128, None, x, 0, x, None, x, ws, None) == want, prec
        assert L.ft_linear_bwd(ctypes.byref(lin), x, x, x, 128, None, x, 0, x, x, x, ws, None) == want, prec
    # a complete 16-bit configuration passes validation (M = 0: nothing runs)
    lin = _linear()
    lin.precision, lin.wd_k, lin.wd_n = 3, x, x
    assert L.ft_linear_fwd(ctypes.byref(lin), x, 0, None, x, 0, x, None, x, ws, None) == FT_OK


def test_dequant_weight_operands_validation(L):
    p = 0x100000
    wk = FtFp4(p, p, p, 256, 512, 1)
    wn = FtFp4(p, p, p, 512, 256, 1)
    assert L.ft_dequant_weight_operands(None, ctypes.byref(wn), p, p, None) == FT_ERR_INVALID_ARG
    assert L.ft_dequant_weight_operands(ctypes.byref(wk), ctypes.byref(wn), None, None, None) == FT_ERR_INVALID_ARG
    assert L.ft_dequant_weight_operands(ctypes.byref(wk), None, None, p, None) == FT_ERR_INVALID_ARG
    bad = FtFp4(p, p, p, 256, 520, 1)
    assert L.ft_dequant_weight_operands(ctypes.byref(bad), None, p, None, None) == FT_ERR_SHAPE
    swapped = FtFp4(p, p, p, 256, 512, 1)
    assert L.ft_dequant_weight_operands(ctypes.byref(wk), ctypes.byref(swapped), None, p, None) == FT_ERR_SHAPE
    assert L.ft_dequant_weight_operands(ctypes.byref(wk), ctypes.byref(wn), p + 8, None, None) == FT_ERR_ALIGN
    empty = FtFp4(p, p, p, 0, 512, 1)
    assert L.ft_dequant_weight_operands(ctypes.byref(empty), None, p, None, None) == FT_OK
