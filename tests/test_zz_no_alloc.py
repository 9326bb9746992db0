"""The few-rows GEMM entry point that allocates no device memory.

fg_fp8_gemm_nt_small_m_no_alloc exists for callers that cannot call cudaMalloc
while they run: a serving engine that reserved nearly all device memory for
its own pool up front, or a latency-critical loop where an allocation (which
may synchronise the device) is not allowed.  It keeps its split-K partial sums
and counters in a device array that the library itself holds, so this test
checks, through the C ABI, that its results match the CPU oracle and what
fg_fp8_gemm_nt gives (within the parity tolerance of the other GPU tests) on
calls made back to back, each reusing the scratch that the previous one left
behind, and that those calls leave the device's free memory unchanged.

The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

DIFF_TOL = 1e-3
MAX_TOL = 1e-2
FG_ERR_UNSUPPORTED = 3

P = ctypes.c_void_p
I = ctypes.c_int


@pytest.fixture(scope="module")
def fg():
    import fp8_fine_grained_tma_b200 as fg
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return fg


@pytest.fixture(scope="module")
def lib(fg):
    lib = ctypes.CDLL(fg.LIB_PATH)
    for name in ("fg_fp8_gemm_nt", "fg_fp8_gemm_nt_small_m_no_alloc"):
        f = getattr(lib, name)
        f.argtypes = [P, P, P, P, P, I, I, I, P]
        f.restype = I
    return lib


def inputs(fg, M, N, K, seed):
    """E4M3 operands with per-block scales (made on the host, uploaded), and
    the CPU oracle's FP64 result for them."""
    import synth
    x = synth.normal_inputs(M, N, K, seed=seed)
    A, B, sfb = x.A.cuda(), x.B.cuda(), x.sfb.cuda()
    sfa = fg.get_col_major_tma_aligned_tensor(x.sfa.cuda())
    ref = oracle.gemm_nt(x.A.numpy(), x.sfa.numpy(), x.B.numpy(), x.sfb.numpy())
    return (A, sfa, B, sfb), ref


def call(fn, ops, D):
    A, sfa, B, sfb = ops
    M, K = A.shape
    N = B.shape[0]
    stream = torch.cuda.current_stream().cuda_stream
    return fn(A.data_ptr(), sfa.data_ptr(), B.data_ptr(), sfb.data_ptr(), D.data_ptr(), M, N, K, stream)


def close(x: torch.Tensor, y):
    """Parity metric of the GPU tests: x (bf16 result) against y (the oracle's
    FP64 result, or another bf16 result)."""
    x = x.double().cpu().numpy()
    y = y.double().cpu().numpy() if isinstance(y, torch.Tensor) else np.asarray(y, dtype=np.float64)
    assert np.all(np.isfinite(x))
    diff = 1.0 - 2.0 * np.sum(x * y) / max(np.sum(x * x + y * y), 1e-300)
    assert diff <= DIFF_TOL, diff
    assert np.max(np.abs(x - y)) <= MAX_TOL * np.max(np.abs(y)), np.max(np.abs(x - y))


# (M, N, K, forced split count or None): the first uses the split plan of the
# normal entry point; the others force several splits, the last more than its
# partial sums can hold, so that the entry point lowers the split count.
CASES = [(64, 2112, 7168, None), (17, 768, 2048, "5"), (200, 1024, 4096, "6"), (256, 4096, 7168, "8")]


@pytest.mark.parametrize("M,N,K,splits", CASES)
def test_no_alloc_matches_the_normal_entry_point(fg, lib, M, N, K, splits, monkeypatch):
    if splits:
        monkeypatch.setenv("FG_FORCE_SPLITS", splits)
    ops, oracle_ref = inputs(fg, M, N, K, seed=20261000 + M)
    other, oracle_other = inputs(fg, 40, 528, 3072, seed=20261999)   # a second shape between the two calls
    ref = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    assert call(lib.fg_fp8_gemm_nt, ops, ref) == 0
    ref_other = torch.empty((40, 528), dtype=torch.bfloat16, device="cuda")
    assert call(lib.fg_fp8_gemm_nt, other, ref_other) == 0
    outs = [torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    out_other = torch.full((40, 528), 7.0, dtype=torch.bfloat16, device="cuda")
    # Warm-up: under CUDA's lazy module loading the first launch of a kernel
    # loads its code into device memory; the calls measured below come after.
    assert call(lib.fg_fp8_gemm_nt_small_m_no_alloc, ops, outs[1]) == 0
    assert call(lib.fg_fp8_gemm_nt_small_m_no_alloc, other, out_other) == 0
    torch.cuda.synchronize()
    outs[1].fill_(7.0)
    out_other.fill_(7.0)
    torch.cuda.synchronize()

    free_before = torch.cuda.mem_get_info()[0]
    assert call(lib.fg_fp8_gemm_nt_small_m_no_alloc, ops, outs[0]) == 0
    assert call(lib.fg_fp8_gemm_nt_small_m_no_alloc, other, out_other) == 0
    assert call(lib.fg_fp8_gemm_nt_small_m_no_alloc, ops, outs[1]) == 0
    torch.cuda.synchronize()
    free_after = torch.cuda.mem_get_info()[0]

    code, detail = fg.get_last_device_status()
    assert code == 0, (code, detail)
    # Each result against the CPU oracle (FP64), and against the normal entry point.
    close(outs[0], oracle_ref)
    close(outs[1], oracle_ref)
    close(out_other, oracle_other)
    close(outs[0], ref)
    close(out_other, ref_other)
    assert torch.equal(outs[0], outs[1])   # the later call ran on the scratch the others left behind
    assert free_after == free_before


def test_no_alloc_rejects_sizes_beyond_its_limits(fg, lib):
    ops, _ = inputs(fg, 64, 256, 256, seed=20261998)
    big_m, _ = inputs(fg, 257, 256, 256, seed=20261997)
    D = torch.empty((257, 256), dtype=torch.bfloat16, device="cuda")
    assert call(lib.fg_fp8_gemm_nt_small_m_no_alloc, big_m, D) == FG_ERR_UNSUPPORTED
    A, sfa, B, sfb = ops
    stream = torch.cuda.current_stream().cuda_stream
    too_wide = 262144 + 16
    assert lib.fg_fp8_gemm_nt_small_m_no_alloc(A.data_ptr(), sfa.data_ptr(), B.data_ptr(), sfb.data_ptr(),
                                               D.data_ptr(), 64, too_wide, 256, stream) == FG_ERR_UNSUPPORTED
