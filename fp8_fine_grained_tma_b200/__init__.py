"""fp8_fine_grained_tma_b200 -- fine-grained-scaled FP8 GEMM for NVIDIA B200.

A thin Python binding over the C ABI of ``libfg8.so`` (declared in
``include/fg8.h``).  It only marshals arguments: torch tensors become device
pointers plus sizes, the current torch stream becomes the launch stream, and
every step of the computation runs in the library's CUDA kernels.  There is no
CPU fallback: if the library is missing, importing this package fails; if no
sm_100 GPU is present, the calls raise.

Entry points (names as in the C ABI without its ``fg_`` prefix):

* ``fp8_gemm_nt(A, sfa, B, sfb, D=None)``
* ``m_grouped_fp8_gemm_nt_contiguous(A, sfa, B, sfb, m_indices, D=None)``
* ``m_grouped_fp8_gemm_nt_masked(A, sfa, B, sfb, masked_m, expected_m=0, D=None)``
* utilities ``set_num_sms``, ``get_num_sms``,
  ``get_m_alignment_for_contiguous_layout``, ``get_tma_aligned_size``,
  ``get_col_major_tma_aligned_tensor`` (deepseek.csdn.net "DeepGEMM：简洁、
  高效…", section "实用工具"), plus ``get_last_device_status`` and
  ``set_wait_limit_ns``.

Operands: E4M3 codes as ``torch.uint8`` or ``torch.float8_e4m3fn`` tensors
(K-major); ``sfa`` in the MN-major TMA-aligned layout made by
``get_col_major_tma_aligned_tensor``; ``sfb`` fp32 ``[ceil(N/128), K/128]``
(``[G, ...]`` for grouped); ``D`` bf16.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfg8.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python fp8_fine_grained_tma_b200/build.py` "
        "(there is no CPU fallback)")

_lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I = ctypes.c_int
_SIG = {
    "fg_status_string": (ctypes.c_char_p, [_I]),
    "fg_version": (ctypes.c_char_p, []),
    "fg_fp8_gemm_nt": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _P]),
    "fg_m_grouped_fp8_gemm_nt_contiguous": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "fg_m_grouped_fp8_gemm_nt_masked": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "fg_get_num_sms": (_I, []),
    "fg_set_num_sms": (_I, [_I]),
    "fg_get_m_alignment_for_contiguous_layout": (_I, []),
    "fg_get_tma_aligned_size": (ctypes.c_size_t, [ctypes.c_size_t, ctypes.c_size_t]),
    "fg_transform_sfa_to_tma_layout": (_I, [_P, _P, _I, _I, _I, _P]),
    "fg_get_last_device_status": (_I, [_P, ctypes.POINTER(_I), ctypes.POINTER(_I)]),
    "fg_set_wait_limit_ns": (_I, [ctypes.c_ulonglong]),
    "fg_get_wait_limit_ns": (ctypes.c_ulonglong, []),
    "fg_query_block_n": (_I, [_I, _I, _I]),
    "fg_query_plan": (_I, [_I, _I, _I, _I, _I, _I] + [ctypes.POINTER(_I)] * 5),
    "fg_jit_compile": (_I, [_I, _I, _I, ctypes.c_char_p, ctypes.c_size_t]),
    "fg_jit_stats": (None, [ctypes.POINTER(_I), ctypes.POINTER(_I), ctypes.POINTER(_I)]),
    "fg_fp8_gemm_nt_small_m_no_alloc": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _P]),
    "fg_quantize_fp8_activations": (_I, [_P, _I, _P, _P, _I, _I, _P]),
}
for _name, (_res, _args) in _SIG.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTED = tuple(_SIG)
BLOCK = 128

FG_OK = 0
FG_ERR_TIMEOUT = 6


class FG8Error(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} ({code})")


def status_string(code: int) -> str:
    return _lib.fg_status_string(code).decode()


def version() -> str:
    return _lib.fg_version().decode()


def _check(code: int, where: str):
    if code != FG_OK:
        raise FG8Error(code, where)


def _stream(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: torch.Tensor) -> int:
    return t.data_ptr()


def _codes(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype not in (torch.uint8, torch.float8_e4m3fn):
        raise TypeError(f"{name} must hold E4M3 codes (uint8 or float8_e4m3fn), got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (K-major)")
    return t


def _f32(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype != torch.float32 or not t.is_cuda:
        raise TypeError(f"{name} must be a float32 CUDA tensor")
    return t


def _check_sfa(sfa: torch.Tensor, groups: int | None, rows: int, kb: int):
    """sfa must be the MN-major TMA-aligned view: [.., rows, KB] with strides
    (.., 1, M_pad) over storage [.., KB, M_pad]."""
    _f32(sfa, "sfa")
    m_pad = get_tma_aligned_size(rows, 4)
    want_shape = (rows, kb) if groups is None else (groups, rows, kb)
    if tuple(sfa.shape) != want_shape:
        raise ValueError(f"sfa shape {tuple(sfa.shape)} != {want_shape}")
    want = (1, m_pad) if groups is None else (kb * m_pad, 1, m_pad)
    if rows > 0 and kb > 0 and tuple(sfa.stride()) != want and not (kb == 1 and sfa.stride()[-2] == 1):
        raise ValueError(f"sfa strides {sfa.stride()} are not the MN-major TMA-aligned layout {want}; "
                         "use get_col_major_tma_aligned_tensor")


def get_num_sms() -> int:
    return _lib.fg_get_num_sms()


def set_num_sms(n: int) -> None:
    _check(_lib.fg_set_num_sms(int(n)), "set_num_sms")


def get_m_alignment_for_contiguous_layout() -> int:
    return _lib.fg_get_m_alignment_for_contiguous_layout()


def get_tma_aligned_size(n: int, elem_bytes: int) -> int:
    r = _lib.fg_get_tma_aligned_size(int(n), int(elem_bytes))
    if r == 0 and n != 0:
        raise ValueError(f"element size {elem_bytes} does not divide 16")
    return r


def get_col_major_tma_aligned_tensor(sfa: torch.Tensor) -> torch.Tensor:
    """Row-major fp32 scales [M, KB] (or [G, M, KB]) -> the same values in the
    MN-major, TMA-aligned layout the GEMMs read: a view of shape [M, KB] with
    strides (1, M_pad) over storage [KB, M_pad] (padding rows are zero)."""
    _f32(sfa, "sfa")
    squeeze = sfa.dim() == 2
    s3 = sfa.unsqueeze(0) if squeeze else sfa
    if s3.dim() != 3:
        raise ValueError("sfa must be [M, KB] or [G, M, KB]")
    s3 = s3.contiguous()
    G, M, KB = s3.shape
    m_pad = get_tma_aligned_size(M, 4)
    storage = torch.empty(G * KB * m_pad, dtype=torch.float32, device=sfa.device)
    with torch.cuda.device(sfa.device):
        _check(_lib.fg_transform_sfa_to_tma_layout(_ptr(s3), _ptr(storage), G, M, KB, _stream()),
               "get_col_major_tma_aligned_tensor")
    out = storage.as_strided((G, M, KB), (KB * m_pad, 1, m_pad))
    return out[0] if squeeze else out


def quantize_fp8_activations(x, stream=None):
    """Row-wise 1x128 block quantisation of activations x [M, K] (float32 or
    bfloat16, K % 128 == 0) into E4M3 codes and FP32 scales, the scales
    already in the MN-major TMA-aligned layout: returns (q uint8 [M, K],
    sfa view [M, K/128] with strides (1, M_pad)), ready for fp8_gemm_nt."""
    if x.dtype not in (torch.float32, torch.bfloat16) or not x.is_cuda or x.dim() != 2:
        raise TypeError("x must be a 2-D float32 or bfloat16 CUDA tensor")
    x = x.contiguous()
    M, K = x.shape
    if K % BLOCK != 0:
        raise ValueError("K must be a multiple of 128")
    KB = K // BLOCK
    m_pad = get_tma_aligned_size(M, 4)
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    storage = torch.empty(max(1, KB * m_pad), dtype=torch.float32, device=x.device)
    with torch.cuda.device(x.device):
        _check(_lib.fg_quantize_fp8_activations(_ptr(x), 1 if x.dtype == torch.bfloat16 else 0, _ptr(q),
                                                _ptr(storage), M, K, _stream(stream)),
               "quantize_fp8_activations")
    return q, storage[:KB * m_pad].as_strided((M, KB), (1, m_pad))


def fp8_gemm_nt(A, sfa, B, sfb, D=None, stream=None):
    """D[M,N] (bf16) = fine-grained-scaled A[M,K] . B[N,K]^T."""
    A = _codes(A, "A")
    B = _codes(B, "B")
    M, K = A.shape
    N = B.shape[0]
    if B.shape[1] != K:
        raise ValueError("A and B disagree on K")
    KB = K // BLOCK
    _check_sfa(sfa, None, M, KB)
    _f32(sfb, "sfb")
    if tuple(sfb.shape) != ((N + BLOCK - 1) // BLOCK, KB) or not sfb.is_contiguous():
        raise ValueError(f"sfb must be contiguous [{(N + BLOCK - 1) // BLOCK}, {KB}]")
    if D is None:
        D = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    elif D.dtype != torch.bfloat16 or tuple(D.shape) != (M, N) or not D.is_contiguous():
        raise ValueError("D must be a contiguous bf16 [M, N] tensor")
    with torch.cuda.device(A.device):
        _check(_lib.fg_fp8_gemm_nt(_ptr(A), _ptr(sfa), _ptr(B), _ptr(sfb), _ptr(D), M, N, K, _stream(stream)),
               "fp8_gemm_nt")
    return D


def fp8_gemm_nt_small_m_no_alloc(A, sfa, B, sfb, D, stream=None):
    """fp8_gemm_nt for 1 <= M <= 256 that allocates no device memory: the
    split-K scratch is a device array the library holds on every GPU it is
    loaded on, so callers whose device memory is all reserved up front, or
    that may not call cudaMalloc in their serving loop, can still split K.
    D (bf16 [M, N]) must be given.  Calls that overlap on the GPU share that
    scratch and race; the first call on a device, which looks up the scratch
    address, should come before any stream capture."""
    A = _codes(A, "A")
    B = _codes(B, "B")
    M, K = A.shape
    N = B.shape[0]
    if B.shape[1] != K:
        raise ValueError("A and B disagree on K")
    KB = K // BLOCK
    _check_sfa(sfa, None, M, KB)
    _f32(sfb, "sfb")
    if tuple(sfb.shape) != ((N + BLOCK - 1) // BLOCK, KB) or not sfb.is_contiguous():
        raise ValueError(f"sfb must be contiguous [{(N + BLOCK - 1) // BLOCK}, {KB}]")
    if D.dtype != torch.bfloat16 or tuple(D.shape) != (M, N) or not D.is_contiguous():
        raise ValueError("D must be a contiguous bf16 [M, N] tensor")
    with torch.cuda.device(A.device):
        _check(_lib.fg_fp8_gemm_nt_small_m_no_alloc(_ptr(A), _ptr(sfa), _ptr(B), _ptr(sfb), _ptr(D), M, N, K,
                                                    _stream(stream)),
               "fp8_gemm_nt_small_m_no_alloc")
    return D


def m_grouped_fp8_gemm_nt_contiguous(A, sfa, B, sfb, m_indices, D=None, stream=None):
    """Contiguous-grouped MoE GEMM: row m of D uses expert m_indices[m]; rows
    tagged -1 are never written."""
    A = _codes(A, "A")
    B = _codes(B, "B")
    M_tot, K = A.shape
    G, N, K2 = B.shape
    if K2 != K:
        raise ValueError("A and B disagree on K")
    KB = K // BLOCK
    _check_sfa(sfa, None, M_tot, KB)
    _f32(sfb, "sfb")
    if tuple(sfb.shape) != (G, (N + BLOCK - 1) // BLOCK, KB) or not sfb.is_contiguous():
        raise ValueError("sfb must be contiguous [G, ceil(N/128), K/128]")
    if m_indices.dtype != torch.int32 or m_indices.numel() != M_tot or not m_indices.is_cuda:
        raise ValueError("m_indices must be an int32 CUDA tensor with one entry per row of A")
    if D is None:
        D = torch.empty((M_tot, N), dtype=torch.bfloat16, device=A.device)
    with torch.cuda.device(A.device):
        _check(_lib.fg_m_grouped_fp8_gemm_nt_contiguous(_ptr(A), _ptr(sfa), _ptr(B), _ptr(sfb), _ptr(D),
                                                        _ptr(m_indices.contiguous()), M_tot, N, K, G,
                                                        _stream(stream)),
               "m_grouped_fp8_gemm_nt_contiguous")
    return D


def m_grouped_fp8_gemm_nt_masked(A, sfa, B, sfb, masked_m, expected_m: int = 0, D=None, stream=None):
    """Masked-grouped MoE GEMM: rows r < masked_m[g] of D[g] are computed, the
    others are never written."""
    A = _codes(A, "A")
    B = _codes(B, "B")
    G, M_max, K = A.shape
    G2, N, K2 = B.shape
    if G2 != G or K2 != K:
        raise ValueError("A and B disagree on G or K")
    KB = K // BLOCK
    _check_sfa(sfa, G, M_max, KB)
    _f32(sfb, "sfb")
    if tuple(sfb.shape) != (G, (N + BLOCK - 1) // BLOCK, KB) or not sfb.is_contiguous():
        raise ValueError("sfb must be contiguous [G, ceil(N/128), K/128]")
    if masked_m.dtype != torch.int32 or masked_m.numel() != G or not masked_m.is_cuda:
        raise ValueError("masked_m must be an int32 CUDA tensor with one entry per group")
    if D is None:
        D = torch.empty((G, M_max, N), dtype=torch.bfloat16, device=A.device)
    with torch.cuda.device(A.device):
        _check(_lib.fg_m_grouped_fp8_gemm_nt_masked(_ptr(A), _ptr(sfa), _ptr(B), _ptr(sfb), _ptr(D),
                                                    _ptr(masked_m.contiguous()), G, M_max, N, K,
                                                    int(expected_m), _stream(stream)),
               "m_grouped_fp8_gemm_nt_masked")
    return D


def get_last_device_status(stream=None):
    """(code, detail) of the first device-side error since the last call
    (0 = none); synchronises the stream and clears the status word."""
    code = ctypes.c_int(0)
    detail = ctypes.c_int(0)
    _check(_lib.fg_get_last_device_status(_stream(stream), ctypes.byref(code), ctypes.byref(detail)),
           "get_last_device_status")
    return code.value, detail.value


def set_wait_limit_ns(ns: int) -> None:
    _check(_lib.fg_set_wait_limit_ns(int(ns)), "set_wait_limit_ns")


def get_wait_limit_ns() -> int:
    return int(_lib.fg_get_wait_limit_ns())


def query_block_n(M: int, N: int, K: int) -> int:
    return _lib.fg_query_block_n(M, N, K)


def query_plan(layout: str, rows: int, N: int, K: int, G: int = 1, expected_m: int = 0) -> dict:
    """Launch plan of a GEMM call (diagnostics): which kernel, its tile width,
    CTA pairs, K splits and cluster size.  layout: "normal", "contiguous" or
    "masked"; rows = M, M_tot or M_max."""
    lay = {"normal": 0, "contiguous": 1, "masked": 2}[layout]
    out = [ctypes.c_int(0) for _ in range(5)]
    _check(_lib.fg_query_plan(lay, int(rows), int(N), int(K), int(G), int(expected_m), *[ctypes.byref(o) for o in out]),
           "query_plan")
    kernel, tile_n, pair, splits, cluster = (o.value for o in out)
    return {"kernel": "decode" if kernel == 1 else "tile", "tile_n": tile_n, "pair": bool(pair), "splits": splits,
            "cluster": cluster}


def jit_compile(block_n: int, pair: bool, k_blocks: int) -> str:
    """Compile (or find in the on-disk cache) the tile kernel specialised for
    (block_n, pair, k_blocks) with NVRTC; returns the cubin's path.  Needs no
    GPU.  The GEMMs use such kernels when FG_JIT=1 is set."""
    buf = ctypes.create_string_buffer(4096)
    _check(_lib.fg_jit_compile(int(block_n), 1 if pair else 0, int(k_blocks), buf, len(buf)), "jit_compile")
    return buf.value.decode()


def jit_stats() -> dict:
    """Runtime specialisations compiled / read from the disk cache by this
    process, and GEMM launches that ran a runtime-compiled kernel."""
    c, d, n = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    _lib.fg_jit_stats(ctypes.byref(c), ctypes.byref(d), ctypes.byref(n))
    return {"compiled": c.value, "loaded_from_disk": d.value, "launches": n.value}
