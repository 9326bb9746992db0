"""C-ABI checks that need no GPU: the library loads, exports every symbol the
public header declares, and rejects bad arguments before touching a device."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fg8.h")


@pytest.fixture(scope="module")
def lib():
    # build.py is loaded by path: importing the package needs the library.
    import importlib.util
    spec = importlib.util.spec_from_file_location("fg8_build", os.path.join(ROOT, "fp8_fine_grained_tma_b200",
                                                                            "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    path = build.build()
    return ctypes.CDLL(path)


def header_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fg_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    syms = header_symbols()
    for name in ["fg_fp8_gemm_nt", "fg_m_grouped_fp8_gemm_nt_contiguous", "fg_m_grouped_fp8_gemm_nt_masked",
                 "fg_get_num_sms", "fg_set_num_sms", "fg_get_m_alignment_for_contiguous_layout",
                 "fg_get_tma_aligned_size", "fg_transform_sfa_to_tma_layout", "fg_get_last_device_status"]:
        assert name in syms


def test_library_exports_every_header_symbol(lib):
    missing = [s for s in header_symbols() if not hasattr(lib, s)]
    assert not missing, missing


def test_binding_exposes_same_names():
    import fp8_fine_grained_tma_b200 as fg
    for s in header_symbols():
        assert s in fg.EXPORTED, s
        py = s[len("fg_"):]
        if py in ("status_string", "version", "get_last_device_status", "set_wait_limit_ns",
                  "get_wait_limit_ns", "query_block_n", "get_num_sms", "set_num_sms",
                  "get_m_alignment_for_contiguous_layout", "get_tma_aligned_size",
                  "fp8_gemm_nt", "m_grouped_fp8_gemm_nt_contiguous", "m_grouped_fp8_gemm_nt_masked",
                  "fp8_gemm_nt_small_m_no_alloc", "quantize_fp8_activations", "query_plan"):
            assert hasattr(fg, py), py
    assert hasattr(fg, "get_col_major_tma_aligned_tensor")


P = ctypes.c_void_p
FAKE = 0x100000  # 16-byte aligned, never dereferenced: every call below fails its checks first


def gemm(lib, A=FAKE, sfa=FAKE, B=FAKE, sfb=FAKE, D=FAKE, M=64, N=128, K=256):
    f = lib.fg_fp8_gemm_nt
    f.argtypes = [P, P, P, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P]
    f.restype = ctypes.c_int
    return f(A, sfa, B, sfb, D, M, N, K, None)


FG_OK, FG_ERR_INVALID_ARG, FG_ERR_ALIGNMENT, FG_ERR_UNSUPPORTED, FG_ERR_NO_DEVICE = 0, 1, 2, 3, 4


def test_gemm_argument_checks(lib):
    assert gemm(lib, K=130) == FG_ERR_UNSUPPORTED
    assert gemm(lib, K=0) == FG_ERR_UNSUPPORTED
    assert gemm(lib, N=120) == FG_ERR_UNSUPPORTED
    assert gemm(lib, M=-1) == FG_ERR_INVALID_ARG
    assert gemm(lib, A=None) == FG_ERR_INVALID_ARG
    assert gemm(lib, D=None) == FG_ERR_INVALID_ARG
    assert gemm(lib, A=FAKE + 8) == FG_ERR_ALIGNMENT
    assert gemm(lib, D=FAKE + 2) == FG_ERR_ALIGNMENT
    assert gemm(lib, sfa=FAKE + 4) == FG_ERR_ALIGNMENT
    assert gemm(lib, sfb=FAKE + 1) == FG_ERR_ALIGNMENT
    assert gemm(lib, M=0, A=None, sfa=None, B=None, sfb=None, D=None) == FG_OK   # empty problem: no-op


@pytest.mark.skipif(torch.cuda.is_available(), reason="fake pointers would be launched on a real device")
def test_valid_arguments_without_device_report_no_device(lib):
    assert gemm(lib) == FG_ERR_NO_DEVICE


def test_grouped_argument_checks(lib):
    c = lib.fg_m_grouped_fp8_gemm_nt_contiguous
    c.argtypes = [P] * 6 + [ctypes.c_int] * 4 + [P]
    c.restype = ctypes.c_int
    assert c(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 200, 128, 256, 2, None) == FG_ERR_INVALID_ARG  # M_tot % 128
    assert c(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 256, 128, 256, 0, None) == FG_ERR_INVALID_ARG  # G == 0
    assert c(FAKE, FAKE, FAKE, FAKE, FAKE, None, 256, 128, 256, 2, None) == FG_ERR_INVALID_ARG  # no tags
    assert c(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 2, 256, 128, 256, 2, None) == FG_ERR_ALIGNMENT
    assert c(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 256, 128, 100, 2, None) == FG_ERR_UNSUPPORTED
    m = lib.fg_m_grouped_fp8_gemm_nt_masked
    m.argtypes = [P] * 6 + [ctypes.c_int] * 5 + [P]
    m.restype = ctypes.c_int
    assert m(FAKE, FAKE, FAKE, FAKE, FAKE, None, 4, 256, 128, 256, 0, None) == FG_ERR_INVALID_ARG
    assert m(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 256, 40, 256, 0, None) == FG_ERR_UNSUPPORTED
    assert m(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 256, 128, 256, -1, None) == FG_ERR_INVALID_ARG
    assert m(None, None, None, None, None, None, 0, 256, 128, 256, 0, None) == FG_OK  # no groups: no-op


def test_no_alloc_argument_checks(lib):
    f = lib.fg_fp8_gemm_nt_small_m_no_alloc
    f.argtypes = [P, P, P, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P]
    f.restype = ctypes.c_int
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 257, 128, 256, None) == FG_ERR_UNSUPPORTED      # M above 256
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 64, 262160, 256, None) == FG_ERR_UNSUPPORTED    # N above 262144
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 64, 128, 200, None) == FG_ERR_UNSUPPORTED
    assert f(FAKE + 8, FAKE, FAKE, FAKE, FAKE, 64, 128, 256, None) == FG_ERR_ALIGNMENT
    assert f(None, FAKE, FAKE, FAKE, FAKE, 64, 128, 256, None) == FG_ERR_INVALID_ARG
    assert f(None, None, None, None, None, 0, 128, 256, None) == FG_OK


def test_quantiser_argument_checks(lib):
    f = lib.fg_quantize_fp8_activations
    f.argtypes = [P, ctypes.c_int, P, P, ctypes.c_int, ctypes.c_int, P]
    f.restype = ctypes.c_int
    assert f(FAKE, 0, FAKE, FAKE, 64, 200, None) == FG_ERR_UNSUPPORTED       # K % 128
    assert f(FAKE, 2, FAKE, FAKE, 64, 256, None) == FG_ERR_INVALID_ARG       # dtype flag
    assert f(FAKE, 0, FAKE, FAKE, -1, 256, None) == FG_ERR_INVALID_ARG
    assert f(None, 0, FAKE, FAKE, 64, 256, None) == FG_ERR_INVALID_ARG
    assert f(FAKE + 4, 0, FAKE, FAKE, 64, 256, None) == FG_ERR_ALIGNMENT
    assert f(None, 0, None, None, 0, 256, None) == FG_OK                     # no rows: no-op


def test_helpers(lib):
    lib.fg_get_tma_aligned_size.restype = ctypes.c_size_t
    lib.fg_get_tma_aligned_size.argtypes = [ctypes.c_size_t, ctypes.c_size_t]
    for n in range(0, 50):
        assert lib.fg_get_tma_aligned_size(n, 4) == -(-n // 4) * 4
        assert lib.fg_get_tma_aligned_size(n, 1) == -(-n // 16) * 16
    assert lib.fg_get_tma_aligned_size(5, 3) == 0
    assert lib.fg_get_m_alignment_for_contiguous_layout() == 128
    lib.fg_set_num_sms.argtypes = [ctypes.c_int]
    assert lib.fg_set_num_sms(0) == FG_ERR_INVALID_ARG
    assert lib.fg_set_num_sms(-3) == FG_ERR_INVALID_ARG
    lib.fg_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    assert lib.fg_set_wait_limit_ns(10) == FG_ERR_INVALID_ARG
    lib.fg_status_string.restype = ctypes.c_char_p
    assert lib.fg_status_string(6) == b"FG_ERR_TIMEOUT"
    t = lib.fg_transform_sfa_to_tma_layout
    t.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P]
    assert t(FAKE, FAKE + 4, 1, 10, 2, None) == FG_ERR_ALIGNMENT
    assert t(None, FAKE, 1, 10, 2, None) == FG_ERR_INVALID_ARG
    assert t(None, None, 1, 0, 2, None) == FG_OK


def test_block_n_choice_is_a_valid_width(lib):
    lib.fg_query_block_n.argtypes = [ctypes.c_int] * 3
    for (M, N, K) in [(64, 2112, 7168), (4096, 24576, 1536), (4096, 7168, 16384), (4096, 4096, 7168),
                      (128, 32768, 512)]:
        bn = abs(lib.fg_query_block_n(M, N, K))   # negative: the tile runs on a CTA pair
        assert 16 <= bn <= 256 and bn % 16 == 0
    assert lib.fg_query_block_n(64, 100, 128) == 0


def test_plan_query_without_a_device():
    """The plan query is host logic: small M goes to the few-rows kernel with
    a token-tile width covering M, larger M to the tile kernel with a block
    width in 16..256; bad arguments are rejected."""
    import fp8_fine_grained_tma_b200 as fg
    p = fg.query_plan("normal", 64, 2112, 7168)
    assert p["kernel"] == "decode" and p["tile_n"] == 64 and 1 <= p["splits"] <= 56
    p = fg.query_plan("normal", 100, 4096, 7168)
    assert p["kernel"] == "decode" and p["tile_n"] == 128
    for layout, rows, G, em in [("normal", 4096, 1, 0), ("contiguous", 37376, 8, 0), ("masked", 256, 32, 128)]:
        p = fg.query_plan(layout, rows, 7168, 2048, G, em)
        assert p["kernel"] == "tile" and 16 <= p["tile_n"] <= 256 and p["tile_n"] % 16 == 0 and p["splits"] == 1
    with pytest.raises(fg.FG8Error):
        fg.query_plan("normal", 64, 2112, 100)
    with pytest.raises(fg.FG8Error):
        fg.query_plan("normal", 0, 2112, 128)


def test_c_program_links_and_checks_the_abi(lib, tmp_path):
    """A plain C program, built with gcc against include/fg8.h and linked to
    libfg8.so, runs the host-side checks without Python in between."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc") or shutil.which("cc")
    if gcc is None:
        pytest.skip("no C compiler")
    libdir = os.path.join(ROOT, "fp8_fine_grained_tma_b200")
    exe = str(tmp_path / "abi_check")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi", "abi_check.c"), "-L", libdir, "-lfg8",
                    "-Wl,-rpath," + libdir, "-o", exe], check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr


def test_binding_rejects_bad_tensors_before_any_launch():
    """The Python binding validates dtypes, devices, shapes and layouts on the
    host and raises before it reaches the library."""
    import fp8_fine_grained_tma_b200 as fg
    A = torch.zeros((64, 256), dtype=torch.uint8)          # CPU tensor
    B = torch.zeros((128, 256), dtype=torch.uint8)
    sfa = torch.zeros((64, 2), dtype=torch.float32)
    sfb = torch.zeros((1, 2), dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA"):
        fg.fp8_gemm_nt(A, sfa, B, sfb)
    with pytest.raises(TypeError, match="E4M3"):
        fg.fp8_gemm_nt(A.float(), sfa, B, sfb)
    with pytest.raises(TypeError):
        fg.quantize_fp8_activations(torch.zeros((4, 128), dtype=torch.float16))
    with pytest.raises(TypeError):
        fg.get_col_major_tma_aligned_tensor(torch.zeros((4, 2), dtype=torch.float64))
    with pytest.raises(ValueError, match="divide 16"):
        fg.get_tma_aligned_size(5, 3)
    assert fg.get_tma_aligned_size(5, 4) == 8
    assert fg.get_m_alignment_for_contiguous_layout() == 128
    assert fg.status_string(6) == "FG_ERR_TIMEOUT"
