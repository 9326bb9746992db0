"""Pins of the CPU oracle against things other than itself (CPU only).

Each test ties one oracle function to an independent fact: torch's
float8_e4m3fn cast (a library routine), a hand-written table of E4M3 values,
numpy float64 matmul of the dequantised operands, closed forms (permutation B,
one isolated scale block), an exact int64 matmul, exact rational arithmetic on
tiny shapes, and the group / mask invariants of the grouped layouts.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- helpers --

def torch_decode(codes) -> np.ndarray:
    """E4M3 codes -> float64 through torch's own float8_e4m3fn cast."""
    t = torch.as_tensor(np.ascontiguousarray(codes, dtype=np.uint8))
    return t.view(torch.float8_e4m3fn).to(torch.float32).to(torch.float64).numpy()


def dequant_ref(A, sfa, B, sfb):
    """numpy float64 matmul of the dequantised operands: a library special case
    of the definition (distributing the block scales over the K sum)."""
    A = np.asarray(A)
    B = np.asarray(B)
    K = A.shape[1]
    N = B.shape[0]
    a = torch_decode(A) * np.repeat(np.asarray(sfa, np.float64), 128, axis=1)[:, :K]
    sfb_rows = np.repeat(np.asarray(sfb, np.float64), 128, axis=0)[:N]
    b = torch_decode(B) * np.repeat(sfb_rows, 128, axis=1)[:, :K]
    return a @ b.T


def rand_problem(M, N, K, seed, scale_lo=-6, scale_hi=6):
    g = torch.Generator().manual_seed(seed)
    A = synth.random_codes((M, K), g).numpy()
    B = synth.random_codes((N, K), g).numpy()
    rng = np.random.default_rng(seed)
    sfa = (rng.uniform(0.5, 2.0, (M, K // 128)) *
           2.0 ** rng.integers(scale_lo, scale_hi, (M, K // 128))).astype(np.float32)
    sfb = (rng.uniform(0.5, 2.0, ((N + 127) // 128, K // 128)) *
           2.0 ** rng.integers(scale_lo, scale_hi, ((N + 127) // 128, K // 128))).astype(np.float32)
    return A, sfa, B, sfb


def assert_close(got, ref, rel=1e-12):
    got = np.asarray(got)
    ref = np.asarray(ref)
    scale = max(1e-300, float(np.max(np.abs(ref))))
    err = float(np.max(np.abs(got - ref)))
    assert err <= rel * scale, f"max err {err} vs scale {scale}"


# ------------------------------------------------------------ E4M3 table --

def test_e4m3_table_matches_torch_cast_all_256_codes():
    tab = oracle.e4m3_table()
    ref = torch_decode(np.arange(256, dtype=np.uint8))
    for c in range(256):
        if math.isnan(ref[c]):
            assert math.isnan(tab[c]), hex(c)
        else:
            assert tab[c] == ref[c], (hex(c), tab[c], ref[c])
            assert math.copysign(1.0, tab[c]) == math.copysign(1.0, ref[c]), hex(c)
    assert [c for c in range(256) if math.isnan(tab[c])] == [0x7F, 0xFF]


def test_e4m3_table_matches_hand_written_golden_values():
    tab = oracle.e4m3_table()
    n = 0
    with open(os.path.join(GOLDEN, "e4m3_special_values.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            code_s, val_s = line.split()[:2]
            code = int(code_s, 16)
            val = float(val_s)
            if math.isnan(val):
                assert math.isnan(tab[code])
            else:
                assert tab[code] == val and math.copysign(1, tab[code]) == math.copysign(1, val), code_s
            n += 1
    assert n >= 20


def test_e4m3_table_is_monotone_and_symmetric():
    tab = oracle.e4m3_table()
    pos = tab[0:0x7F]
    assert np.all(np.diff(pos) > 0)
    assert pos.max() == 448.0
    for c in range(0x7F):
        assert tab[c | 0x80] == -tab[c]


# ------------------------------------------------------------ normal GEMM --

@pytest.mark.parametrize("M,N,K,seed", [(1, 16, 128, 1), (7, 200, 256, 2), (33, 2112 // 8, 384, 3),
                                         (130, 144, 512, 4)])
def test_gemm_matches_numpy_dequantised_matmul(M, N, K, seed):
    A, sfa, B, sfb = rand_problem(M, N, K, seed)
    D = oracle.gemm_nt(A, sfa, B, sfb)
    assert_close(D, dequant_ref(A, sfa, B, sfb))


def test_gemm_on_quantised_normal_inputs_matches_numpy():
    x = synth.normal_inputs(64, 264, 768, seed=synth.seed_for(0, 9))
    A, sfa, B, sfb = (t.numpy() for t in (x.A, x.sfa, x.B, x.sfb))
    assert_close(oracle.gemm_nt(A, sfa, B, sfb), dequant_ref(A, sfa, B, sfb))


def test_gemm_row_subset_equals_full_rows():
    A, sfa, B, sfb = rand_problem(40, 96, 256, 5)
    full = oracle.gemm_nt(A, sfa, B, sfb)
    rows = [39, 0, 17, 17, 5]
    sub = oracle.gemm_nt(A, sfa, B, sfb, rows=rows)
    assert np.array_equal(sub, full[rows])


def test_gemm_permutation_b_closed_form():
    """B = permutation matrix (code 0x38 = 1.0), sfb = 1: D[m,n] = dec(A[m,p(n)]) * sfa[m, p(n)//128]."""
    M, K = 9, 256
    N = K
    rng = np.random.default_rng(7)
    perm = rng.permutation(K)
    g = torch.Generator().manual_seed(7)
    A = synth.random_codes((M, K), g).numpy()
    B = np.zeros((N, K), dtype=np.uint8)
    B[np.arange(N), perm] = 0x38
    sfa = (2.0 ** rng.integers(-4, 4, (M, K // 128))).astype(np.float32) * np.float32(1.5)
    sfb = np.ones((N // 128, K // 128), dtype=np.float32)
    D = oracle.gemm_nt(A, sfa, B, sfb)
    decA = torch_decode(A)
    expect = decA[:, perm] * sfa[:, perm // 128].astype(np.float64)
    assert np.array_equal(D, expect)


def test_gemm_integer_inputs_exact_against_int64_matmul():
    """Codes for {-2,-1,0,1,2}, power-of-two scales constant along K: the
    result is an exact dyadic rational, equal to an int64 matmul scaled."""
    M, N, K = 24, 272, 640
    rng = np.random.default_rng(11)
    vals = np.array([-2, -1, 0, 1, 2])
    codes = {-2: 0xC0, -1: 0xB8, 0: 0x00, 1: 0x38, 2: 0x40}
    Ai = rng.choice(vals, (M, K))
    Bi = rng.choice(vals, (N, K))
    A = np.vectorize(codes.get)(Ai).astype(np.uint8)
    B = np.vectorize(codes.get)(Bi).astype(np.uint8)
    ea = rng.integers(-5, 5, M)
    eb = rng.integers(-5, 5, (N + 127) // 128)
    sfa = np.repeat((2.0 ** ea)[:, None], K // 128, axis=1).astype(np.float32)
    sfb = np.repeat((2.0 ** eb)[:, None], K // 128, axis=1).astype(np.float32)
    D = oracle.gemm_nt(A, sfa, B, sfb)
    P = Ai.astype(np.int64) @ Bi.astype(np.int64).T
    expect = P * (2.0 ** ea)[:, None] * (2.0 ** eb[np.arange(N) // 128])[None, :]
    assert np.array_equal(D, expect)


def test_gemm_single_scale_block_isolated():
    """All sfa zero except (m0, kb0): only row m0 is non-zero, and it equals
    that block's dot products times its two scales."""
    M, N, K = 6, 160, 512
    A, sfa, B, sfb = rand_problem(M, N, K, 13)
    m0, kb0 = 4, 2
    sfa2 = np.zeros_like(sfa)
    sfa2[m0, kb0] = sfa[m0, kb0]
    D = oracle.gemm_nt(A, sfa2, B, sfb)
    assert np.all(D[np.arange(M) != m0] == 0.0)
    blk = slice(kb0 * 128, (kb0 + 1) * 128)
    part = torch_decode(A[m0, blk]) @ torch_decode(B[:, blk]).T
    expect = part * float(sfa[m0, kb0]) * sfb[np.arange(N) // 128, kb0].astype(np.float64)
    assert_close(D[m0], expect, rel=1e-15)


def test_gemm_exact_rational_brute_force_tiny():
    M, N, K = 3, 5, 256
    A, sfa, B, sfb = rand_problem(M, N, K, 17)
    D = oracle.gemm_nt(A, sfa, B, sfb)
    da = torch_decode(A)
    db = torch_decode(B)
    for m in range(M):
        for n in range(N):
            tot = Fraction(0)
            for k in range(K):
                tot += (Fraction(da[m, k]) * Fraction(float(sfa[m, k // 128])) *
                        Fraction(db[n, k]) * Fraction(float(sfb[n // 128, k // 128])))
            exact = float(tot)
            assert abs(D[m, n] - exact) <= 1e-15 * max(1.0, abs(exact)) * 4


def test_gemm_doubling_sfa_doubles_d_exactly():
    A, sfa, B, sfb = rand_problem(8, 48, 384, 19)
    D1 = oracle.gemm_nt(A, sfa, B, sfb)
    D2 = oracle.gemm_nt(A, sfa * 2, B, sfb)
    assert np.array_equal(D2, 2 * D1)


def test_gemm_rejects_k_not_multiple_of_128():
    A = np.zeros((2, 130), np.uint8)
    with pytest.raises(Exception):
        oracle.gemm_nt(A, np.ones((2, 1), np.float32), np.zeros((16, 130), np.uint8),
                       np.ones((1, 1), np.float32))


# ---------------------------------------------------------- grouped GEMMs --

def test_contiguous_equals_per_expert_normal_gemm():
    G, N, K = 3, 192, 256
    x = synth.contiguous_inputs(G, N, K, seed=23, counts=[5, 0, 130])
    A, sfa, B, sfb, mi = (t.numpy() for t in (x.A, x.sfa, x.B, x.sfb, x.m_indices))
    assert A.shape[0] == 128 + 0 + 256
    D, written = oracle.m_grouped_contiguous(A, sfa, B, sfb, mi)
    assert np.array_equal(written, mi >= 0)
    assert np.all(np.isnan(D[~written]))
    for e in range(G):
        rows = np.nonzero(mi == e)[0]
        if len(rows) == 0:
            continue
        assert_close(D[rows], dequant_ref(A[rows], sfa[rows], B[e], sfb[e]))


def test_contiguous_all_padding_block_and_out_of_range_tags_not_written():
    G, N, K = 2, 64, 128
    x = synth.contiguous_inputs(G, N, K, seed=29, counts=[100, 40])
    mi = x.m_indices.numpy().copy()
    mi[140:150] = 7  # out of range tag: treated as padding
    D, written = oracle.m_grouped_contiguous(x.A.numpy(), x.sfa.numpy(), x.B.numpy(),
                                             x.sfb.numpy(), mi)
    assert not written[140:150].any()
    assert written[:100].all() and not written[100:128].any()


def test_masked_equals_per_group_normal_gemm_on_first_rows():
    G, M_max, N, K = 4, 200, 144, 384
    x = synth.masked_inputs(G, M_max, N, K, seed=31, masked=[0, 1, 200, 250])
    A, sfa, B, sfb, mm = (t.numpy() for t in (x.A, x.sfa, x.B, x.sfb, x.masked_m))
    D, written = oracle.m_grouped_masked(A, sfa, B, sfb, mm)
    D = D.reshape(G, M_max, N)
    written = written.reshape(G, M_max)
    for g in range(G):
        lim = min(int(mm[g]), M_max)
        assert written[g, :lim].all() and not written[g, lim:].any()
        assert np.all(np.isnan(D[g, lim:]))
        if lim:
            assert_close(D[g, :lim], dequant_ref(A[g, :lim], sfa[g, :lim], B[g], sfb[g]))


def test_masked_row_subset():
    G, M_max, N, K = 3, 16, 32, 128
    x = synth.masked_inputs(G, M_max, N, K, seed=37, masked=[3, 16, 9])
    args = [t.numpy() for t in (x.A, x.sfa, x.B, x.sfb, x.masked_m)]
    full, wf = oracle.m_grouped_masked(*args)
    rows = [0, 2, 3, 20, 47, 40, 41]
    sub, ws = oracle.m_grouped_masked(*args, rows=rows)
    assert np.array_equal(ws, wf[rows])
    assert np.array_equal(sub[ws], full[rows][ws])


# ------------------------------------------------- layout helpers, quantiser --

def test_tma_aligned_size_closed_form():
    for n in range(0, 70):
        assert oracle.tma_aligned_size(n, 4) == -(-n // 4) * 4
        assert oracle.tma_aligned_size(n, 2) == -(-n // 8) * 8
        assert oracle.tma_aligned_size(n, 1) == -(-n // 16) * 16


def test_sfa_transform_is_transpose_with_zero_padding():
    rng = np.random.default_rng(41)
    s = rng.standard_normal((3, 37, 5)).astype(np.float32)
    out = oracle.sfa_to_mn_major(s)
    assert out.shape == (3, 5, 40)
    assert np.array_equal(out[:, :, :37], np.transpose(s, (0, 2, 1)))
    assert np.all(out[:, :, 37:] == 0)
    out2 = oracle.sfa_to_mn_major(s[0])
    assert np.array_equal(out2, out[0])


def test_e4m3_encode_ties_and_saturation():
    assert oracle.e4m3_encode(1.0625) == 0x38      # tie 1.0 / 1.125 -> even code
    assert oracle.e4m3_encode(1.1875) == 0x3A      # tie 1.125 / 1.25 -> even code 0x3A
    assert oracle.e4m3_encode(2.0 ** -10) == 0x00  # half the smallest subnormal -> 0
    assert oracle.e4m3_encode(3 * 2.0 ** -10) == 0x02
    assert oracle.e4m3_encode(448.5) == 0x7E
    assert oracle.e4m3_encode(1e9) == 0x7E
    assert oracle.e4m3_encode(-1e9) == 0xFE
    assert oracle.e4m3_encode(-0.0) == 0x80
    for v in [1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10, 300.0, -17.3, 0.0123]:
        t = torch.tensor([v], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)
        assert oracle.e4m3_encode(v) == int(t[0]), v


@pytest.mark.parametrize("br", [1, 128])
def test_quantiser_matches_torch_cast(br):
    g = torch.Generator().manual_seed(43)
    x = torch.randn((150, 300), generator=g) * 3
    x[5, :] = 0.0  # all-zero block: amax floor
    q_ref, s_ref = synth._quantize_chunk(x, br)
    q, s = oracle.quantize_blocks(x.numpy(), br)
    assert np.array_equal(s, s_ref.numpy())
    assert np.array_equal(q, q_ref.numpy())


def test_compare_metric_properties():
    y = np.arange(1, 10, dtype=np.float64)
    assert oracle.compare(y, y)["diff"] == 0.0
    c = oracle.compare(-y, y)
    assert abs(c["diff"] - 2.0) < 1e-15
    c = oracle.compare(y * 1.01, y)
    assert 0 < c["diff"] < 1e-4


# ------------------------------------------------------ randomised sweep --

from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=25, deadline=None)
@given(M=st.integers(1, 40), nblk=st.integers(1, 3), N16=st.integers(1, 20), seed=st.integers(0, 2**31 - 1))
def test_gemm_random_shapes_match_numpy(M, nblk, N16, seed):
    """Random ragged shapes (M any, N any multiple of 16, K up to 3 blocks)
    and random scales over many binades: the oracle equals the numpy float64
    matmul of the dequantised operands."""
    K, N = 128 * nblk, 16 * N16
    A, sfa, B, sfb = rand_problem(M, N, K, seed)
    assert_close(oracle.gemm_nt(A, sfa, B, sfb), dequant_ref(A, sfa, B, sfb))


def test_synthetic_inputs_are_deterministic():
    """The same seed gives the same bytes and scales (every parity test and
    the bench rely on regenerating inputs on both sides)."""
    a = synth.normal_inputs(33, 144, 256, seed=123)
    b = synth.normal_inputs(33, 144, 256, seed=123)
    c = synth.normal_inputs(33, 144, 256, seed=124)
    for k in ("A", "sfa", "B", "sfb"):
        assert torch.equal(getattr(a, k), getattr(b, k))
    assert not torch.equal(a.A, c.A)
