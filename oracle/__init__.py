"""CPU oracle for the fine-grained-scaled FP8 GEMM (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  It shares
no code with the CUDA library: the arithmetic lives in ``fg8_oracle.c``
(plain C, FP64 accumulation, OpenMP over output elements), compiled here with
gcc and called through ctypes on numpy arrays.

What each function computes, and the pages it follows, is stated in
``fg8_oracle.c``.  In short (DeepSeek-V3-style fine-grained scaling, chujupifa.com
"机器之心报道" opening summary; E4M3 format, ai.abqq.net "DeepSeek开源周第三天…
DeepGEMM：FP8" section 3)::

    D[m,n] = sum_kb (sum_{k in kb} dec(A[m,k]) dec(B[n,k])) sfa[m,kb] sfb[n//128,kb]

Pins (tests/test_oracle.py): all 256 E4M3 codes against torch's float8_e4m3fn
cast and a hand-written table of special values; numpy float64 matmul of the
dequantised operands; permutation-B closed form; integer-valued inputs against
an exact int64 matmul; single-block isolation; exact rational brute force;
group and mask invariants; the scale-layout transform against a transpose; the
quantiser against torch's cast.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fg8_oracle.c")
_LIB = os.path.join(_HERE, "libfg8_oracle.so")
_lock = threading.Lock()
_lib = None

BLOCK = 128


def build(force: bool = False) -> str:
    """Compile fg8_oracle.c into libfg8_oracle.so (gcc, -O2, OpenMP, no fast-math)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        build()
        lib = ctypes.CDLL(_LIB)
        p = ctypes.c_void_p
        i = ctypes.c_int
        lib.fg8o_e4m3_table.argtypes = [p]
        lib.fg8o_e4m3_table.restype = None
        lib.fg8o_num_threads.argtypes = []
        lib.fg8o_num_threads.restype = i
        lib.fg8o_gemm_nt.argtypes = [p, p, p, p, i, i, i, p, i, p, i]
        lib.fg8o_gemm_nt.restype = i
        lib.fg8o_m_grouped_contiguous.argtypes = [p, p, p, p, p, i, i, i, i, p, i, p, p, i]
        lib.fg8o_m_grouped_contiguous.restype = i
        lib.fg8o_m_grouped_masked.argtypes = [p, p, p, p, p, i, i, i, i, p, i, p, p, i]
        lib.fg8o_m_grouped_masked.restype = i
        lib.fg8o_tma_aligned_size.argtypes = [ctypes.c_longlong, ctypes.c_longlong]
        lib.fg8o_tma_aligned_size.restype = ctypes.c_longlong
        lib.fg8o_sfa_to_mn_major.argtypes = [p, p, i, i, i]
        lib.fg8o_sfa_to_mn_major.restype = i
        lib.fg8o_e4m3_encode.argtypes = [ctypes.c_float]
        lib.fg8o_e4m3_encode.restype = ctypes.c_uint8
        lib.fg8o_quantize_blocks.argtypes = [p, i, i, i, p, p]
        lib.fg8o_quantize_blocks.restype = i
        _lib = lib
        return lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags.c_contiguous
    return a.ctypes.data_as(ctypes.c_void_p)


def _u8(a) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype != np.uint8:
        a = a.view(np.uint8) if a.itemsize == 1 else a.astype(np.uint8)
    return np.ascontiguousarray(a)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def num_threads() -> int:
    return _load().fg8o_num_threads()


def e4m3_table() -> np.ndarray:
    """256 doubles: the real value of every E4M3 code (NaN for 0x7F, 0xFF)."""
    out = np.empty(256, dtype=np.float64)
    _load().fg8o_e4m3_table(_ptr(out))
    return out


def e4m3_encode(x: float) -> int:
    return int(_load().fg8o_e4m3_encode(float(x)))


def gemm_nt(A, sfa, B, sfb, rows=None, threads: int = 0) -> np.ndarray:
    """Normal GEMM.  A [M,K] codes, sfa [M,K/128] fp32 row-major, B [N,K] codes,
    sfb [ceil(N/128),K/128] fp32.  Returns D[rows, :] as float64 (all rows when
    ``rows`` is None)."""
    A, B, sfa, sfb = _u8(A), _u8(B), _f32(sfa), _f32(sfb)
    M, K = A.shape
    N = B.shape[0]
    KB = K // BLOCK
    assert B.shape == (N, K) and sfa.shape == (M, KB)
    assert sfb.shape == ((N + BLOCK - 1) // BLOCK, KB)
    r = None if rows is None else _i32(rows)
    n_rows = M if r is None else len(r)
    D = np.empty((n_rows, N), dtype=np.float64)
    rc = _load().fg8o_gemm_nt(_ptr(A), _ptr(sfa), _ptr(B), _ptr(sfb), M, N, K,
                              _ptr(r), n_rows, _ptr(D), threads)
    if rc != 0:
        raise ValueError(f"fg8o_gemm_nt: bad sizes M={M} N={N} K={K}")
    return D


def m_grouped_contiguous(A, sfa, B, sfb, m_indices, rows=None, threads: int = 0):
    """Contiguous-grouped GEMM.  A [M_tot,K], sfa [M_tot,K/128], B [G,N,K],
    sfb [G,ceil(N/128),K/128], m_indices int32 [M_tot] (-1 = padding).
    Returns (D[rows, :] float64 with NaN on unwritten rows, written bool[rows])."""
    A, B, sfa, sfb, mi = _u8(A), _u8(B), _f32(sfa), _f32(sfb), _i32(m_indices)
    M_tot, K = A.shape
    G, N, _ = B.shape
    r = None if rows is None else _i32(rows)
    n_rows = M_tot if r is None else len(r)
    D = np.full((n_rows, N), np.nan, dtype=np.float64)
    written = np.zeros(n_rows, dtype=np.uint8)
    rc = _load().fg8o_m_grouped_contiguous(_ptr(A), _ptr(sfa), _ptr(B), _ptr(sfb),
                                           _ptr(mi), M_tot, N, K, G, _ptr(r), n_rows,
                                           _ptr(D), _ptr(written), threads)
    if rc != 0:
        raise ValueError("fg8o_m_grouped_contiguous: bad sizes")
    return D, written.astype(bool)


def m_grouped_masked(A, sfa, B, sfb, masked_m, rows=None, threads: int = 0):
    """Masked-grouped GEMM.  A [G,M_max,K], sfa [G,M_max,K/128], B [G,N,K],
    sfb [G,ceil(N/128),K/128], masked_m int32 [G].  ``rows`` are flat ids
    g*M_max + r.  Returns (D float64 [n_rows,N] with NaN on unwritten rows,
    written bool [n_rows])."""
    A, B, sfa, sfb, mm = _u8(A), _u8(B), _f32(sfa), _f32(sfb), _i32(masked_m)
    G, M_max, K = A.shape
    N = B.shape[1]
    r = None if rows is None else _i32(rows)
    n_rows = G * M_max if r is None else len(r)
    D = np.full((n_rows, N), np.nan, dtype=np.float64)
    written = np.zeros(n_rows, dtype=np.uint8)
    rc = _load().fg8o_m_grouped_masked(_ptr(A), _ptr(sfa), _ptr(B), _ptr(sfb),
                                       _ptr(mm), G, M_max, N, K, _ptr(r), n_rows,
                                       _ptr(D), _ptr(written), threads)
    if rc != 0:
        raise ValueError("fg8o_m_grouped_masked: bad sizes")
    return D, written.astype(bool)


def tma_aligned_size(n: int, elem_bytes: int) -> int:
    return int(_load().fg8o_tma_aligned_size(n, elem_bytes))


def sfa_to_mn_major(sfa) -> np.ndarray:
    """[M,KB] or [G,M,KB] fp32 -> [KB,M_pad] or [G,KB,M_pad], zero padded."""
    sfa = _f32(sfa)
    squeeze = sfa.ndim == 2
    s3 = sfa[None] if squeeze else sfa
    G, M, KB = s3.shape
    M_pad = tma_aligned_size(M, 4)
    out = np.empty((G, KB, M_pad), dtype=np.float32)
    rc = _load().fg8o_sfa_to_mn_major(_ptr(np.ascontiguousarray(s3)), _ptr(out), G, M, KB)
    if rc != 0:
        raise ValueError("fg8o_sfa_to_mn_major: bad sizes")
    return out[0] if squeeze else out


def quantize_blocks(x, block_rows: int):
    """x [R,C] fp32 -> (codes uint8 [R,C], scales fp32 [ceil(R/br), ceil(C/128)])."""
    x = _f32(x)
    R, C = x.shape
    q = np.empty((R, C), dtype=np.uint8)
    s = np.empty(((R + block_rows - 1) // block_rows, (C + BLOCK - 1) // BLOCK), dtype=np.float32)
    rc = _load().fg8o_quantize_blocks(_ptr(x), R, C, block_rows, _ptr(q), _ptr(s))
    if rc != 0:
        raise ValueError("fg8o_quantize_blocks: bad sizes")
    return q, s


def compare(gpu, ref) -> dict:
    """Per-tensor agreement in FP64 over the given (written) elements:
    diff = 1 - 2 sum(xy) / sum(x^2 + y^2) and max|x - y| / max|y|."""
    x = np.asarray(gpu, dtype=np.float64).ravel()
    y = np.asarray(ref, dtype=np.float64).ravel()
    denom = float(np.sum(x * x + y * y))
    diff = 0.0 if denom == 0.0 else 1.0 - 2.0 * float(np.sum(x * y)) / denom
    ymax = float(np.max(np.abs(y))) if y.size else 0.0
    err = float(np.max(np.abs(x - y))) if y.size else 0.0
    return {"diff": diff, "max_abs_err": err, "max_abs_ref": ymax,
            "rel_max_err": 0.0 if ymax == 0.0 else err / ymax}
