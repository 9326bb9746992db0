"""GPU parity of the activation quantiser against the oracle's block quantiser.

Codes and scales are decided in FP32 on both sides (the same amax, the same
FP32 division and round-to-nearest-even conversion), so they must agree bit
for bit; the MN-major scale layout must equal the oracle's transpose with
zero padding.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fg():
    import fp8_fine_grained_tma_b200 as fg
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return fg


def run_and_compare(fg, x: torch.Tensor):
    M, K = x.shape
    q, sfa = fg.quantize_fp8_activations(x.cuda())
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.quantize_blocks(x.float().numpy(), 1)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    m_pad = fg.get_tma_aligned_size(M, 4)
    KB = K // 128
    storage = torch.as_strided(sfa, (KB, m_pad), (m_pad, 1)).cpu().numpy()
    assert np.array_equal(storage.view(np.uint32), oracle.sfa_to_mn_major(s_ref).view(np.uint32))
    return q, sfa


@pytest.mark.parametrize("M,K", [(1, 128), (3, 256), (17, 1536), (128, 7168), (1000, 512), (4096, 2048)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_quantiser_matches_oracle(fg, M, K, dtype):
    g = torch.Generator().manual_seed(1000 + M + K)
    x = (torch.randn((M, K), generator=g) * 4.0).to(dtype)
    run_and_compare(fg, x)


def test_quantiser_special_blocks(fg):
    """An all-zero block (scale floor), a block with one huge value (everything
    else underflows toward zero and subnormals), negative zeros, and values
    whose quotient lands exactly on ties between E4M3 codes."""
    x = torch.randn((8, 512), generator=torch.Generator().manual_seed(7))
    x[0, :128] = 0.0
    x[1, 128:256] = 1e-3
    x[1, 130] = 3e4
    x[2, :] = -0.0
    x[3, :128] = torch.tensor([448.0, 1.0, 1.0625, 1.1875, 0.0009765625, 17.0, -17.0, 2.5] * 16)
    x[4, 256:384] = 1e-6                     # amax below the 1e-4 floor
    run_and_compare(fg, x)


def e4m3_positive_values():
    """Every finite positive E4M3 value, from the format's definition (bias
    7, subnormals m/8 * 2^-6), in increasing order."""
    vals = [m / 8.0 * 2.0 ** -6 for m in range(1, 8)]
    vals += [(1 + m / 8.0) * 2.0 ** (e - 7) for e in range(1, 16) for m in range(8) if not (e == 15 and m == 7)]
    return np.array(sorted(vals))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_quantiser_rounding_boundaries(fg, dtype):
    """Quotients x / scale within a few FP32 units in the last place of every
    rounding boundary of E4M3 (the midpoint between two neighbouring codes),
    on both sides and at the boundary itself, for blocks with many different
    scales: the codes must equal the oracle's, which divides in IEEE FP32."""
    rng = np.random.default_rng(11)
    vals = e4m3_positive_values()
    mids = (vals[:-1] + vals[1:]) / 2.0
    mids = np.concatenate([[vals[0] / 2.0], mids])          # the boundary between 0 and the smallest code
    offs = np.array([-3, -2, -1, 0, 1, 2, 3], dtype=np.float64) * 2.0 ** -23
    targets = (mids[:, None] * (1.0 + offs[None, :])).reshape(-1)
    rows = []
    for _ in range(64):
        amax = np.float32(np.exp(rng.uniform(np.log(1e-3), np.log(1e3))))
        scale = np.float32(max(amax, np.float32(1e-4))) / np.float32(448.0)
        t = rng.choice(targets, 127)
        sign = rng.choice([-1.0, 1.0], 127)
        body = (sign * t).astype(np.float64) * np.float64(scale)
        block = np.concatenate([[amax], np.clip(body, -amax, amax)]).astype(np.float32)
        rows.append(block[rng.permutation(128)])
    x = torch.from_numpy(np.stack(rows).reshape(8, 8 * 128))
    run_and_compare(fg, x.to(dtype))


def test_quantised_activations_feed_the_gemm(fg):
    """Quantising on the GPU and then multiplying gives the GEMM of the
    oracle's own quantisation of the same activations."""
    M, N, K = 200, 384, 1024
    g = torch.Generator().manual_seed(11)
    xa = torch.randn((M, K), generator=g)
    wb = synth.normal_inputs(8, N, K, seed=12)                   # B operand and its scales
    q, sfa = fg.quantize_fp8_activations(xa.cuda())
    D = fg.fp8_gemm_nt(q, sfa, wb.B.cuda(), wb.sfb.cuda())
    torch.cuda.synchronize()
    qa, sa = oracle.quantize_blocks(xa.numpy(), 1)
    ref = oracle.gemm_nt(qa, sa, wb.B.numpy(), wb.sfb.numpy())
    c = oracle.compare(D.double().cpu().numpy(), ref)
    assert c["diff"] <= 1e-3 and c["rel_max_err"] <= 1e-2, c
