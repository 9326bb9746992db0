"""GPU parity: the CUDA path (through the C ABI binding) against the CPU oracle.

Tolerance (per tensor, over written rows, in FP64):
    1 - 2 sum(xy) / sum(x^2 + y^2) <= 1e-3   and   max|x - y| <= 1e-2 * max|y|.
Rows the GEMM must not write (padding rows tagged -1, rows past masked_m) are
pre-filled with a sentinel and must come back bit-identical.  Cases whose
exact result is representable in BF16 (permutation B, small integers) must be
bit-exact.
"""
import os

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

DIFF_TOL = 1e-3
MAX_TOL = 1e-2
SENTINEL = -12345.0  # exactly representable in bf16 (0xC640 pattern after rounding is fixed below)


@pytest.fixture(scope="module")
def fg():
    import fp8_fine_grained_tma_b200 as fg
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return fg


@pytest.fixture(autouse=True)
def clean_status(fg):
    fg.get_last_device_status()
    yield
    code, detail = fg.get_last_device_status()
    assert code == 0, f"device status {code} detail {detail:#x}"


def check(gpu_rows: np.ndarray, ref_rows: np.ndarray):
    c = oracle.compare(gpu_rows, ref_rows)
    assert np.all(np.isfinite(gpu_rows))
    assert c["diff"] <= DIFF_TOL, c
    assert c["rel_max_err"] <= MAX_TOL, c
    return c


def bf16_of(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16)


def sentinel_bf16():
    return torch.tensor(SENTINEL, dtype=torch.bfloat16)


def to_gpu_normal(fg, x):
    A = x.A.cuda()
    B = x.B.cuda()
    sfa = fg.get_col_major_tma_aligned_tensor(x.sfa.cuda())
    sfb = x.sfb.cuda()
    return A, sfa, B, sfb


# --------------------------------------------------------------- helpers --

def test_sfa_transform_matches_oracle(fg):
    g = torch.Generator().manual_seed(5)
    for G, M, KB in [(1, 37, 5), (3, 256, 56), (2, 1, 1), (1, 4096, 12)]:
        s = torch.randn((G, M, KB), generator=g)
        out = fg.get_col_major_tma_aligned_tensor(s.cuda())
        m_pad = fg.get_tma_aligned_size(M, 4)
        storage = torch.as_strided(out, (G, KB, m_pad), (KB * m_pad, m_pad, 1)).cpu().numpy()
        assert np.array_equal(storage, oracle.sfa_to_mn_major(s.numpy()))
        assert torch.equal(out.cpu(), s)


# ----------------------------------------------------------- normal GEMM --

@pytest.mark.parametrize("M,N,K", [(128, 128, 128), (1, 16, 128), (200, 272, 512), (257, 2112, 1024),
                                   (64, 2112, 7168), (383, 4096, 256)])
def test_normal_gemm_matches_oracle(fg, M, N, K):
    x = synth.normal_inputs(M, N, K, seed=synth.seed_for(0, 50) + M + N)
    A, sfa, B, sfb = to_gpu_normal(fg, x)
    D = fg.fp8_gemm_nt(A, sfa, B, sfb)
    torch.cuda.synchronize()
    ref = oracle.gemm_nt(x.A.numpy(), x.sfa.numpy(), x.B.numpy(), x.sfb.numpy())
    check(D.double().cpu().numpy(), ref)


@pytest.mark.parametrize("pair", [0, 1])
@pytest.mark.parametrize("bn", list(range(16, 257, 16)))
def test_every_block_width_matches_oracle(fg, bn, pair, monkeypatch):
    if pair and bn < 32:
        pytest.skip("CTA pairs start at block width 32")
    monkeypatch.setenv("FG_FORCE_BLOCK_N", str(bn))
    monkeypatch.setenv("FG_FORCE_PAIR", str(pair))
    M, N, K = 300, 400, 384   # ragged M and N, several K blocks, tiles straddling scale blocks
    x = synth.normal_inputs(M, N, K, seed=synth.seed_for(0, 60) + bn)
    A, sfa, B, sfb = to_gpu_normal(fg, x)
    D = fg.fp8_gemm_nt(A, sfa, B, sfb)
    torch.cuda.synchronize()
    ref = oracle.gemm_nt(x.A.numpy(), x.sfa.numpy(), x.B.numpy(), x.sfb.numpy())
    check(D.double().cpu().numpy(), ref)


@pytest.mark.parametrize("bn,pair", [(16, 0), (112, 0), (256, 0), (32, 1), (112, 1), (256, 1)])
def test_permutation_b_is_bit_exact(fg, bn, pair, monkeypatch):
    monkeypatch.setenv("FG_FORCE_BLOCK_N", str(bn))
    monkeypatch.setenv("FG_FORCE_PAIR", str(pair))
    M, K = 130, 384
    N = K
    rng = np.random.default_rng(3)
    perm = rng.permutation(K)
    g = torch.Generator().manual_seed(3)
    A = synth.random_codes((M, K), g).numpy()
    B = np.zeros((N, K), dtype=np.uint8)
    B[np.arange(N), perm] = 0x38
    sfa = (2.0 ** rng.integers(-3, 4, (M, K // 128))).astype(np.float32)
    sfb = np.ones((N // 128, K // 128), dtype=np.float32)
    ref = oracle.gemm_nt(A, sfa, B, sfb)
    D = fg.fp8_gemm_nt(torch.from_numpy(A).cuda(), fg.get_col_major_tma_aligned_tensor(torch.from_numpy(sfa).cuda()),
                       torch.from_numpy(B).cuda(), torch.from_numpy(sfb).cuda())
    assert torch.equal(D.cpu().view(torch.int16), bf16_of(ref).view(torch.int16))


def test_integer_inputs_are_bit_exact(fg):
    M, N, K = 256, 320, 256
    rng = np.random.default_rng(4)
    code = {-1: 0xB8, 0: 0x00, 1: 0x38}
    Ai = rng.choice([-1, 0, 1], (M, K))
    Bi = rng.choice([-1, 0, 1], (N, K))
    A = np.vectorize(code.get)(Ai).astype(np.uint8)
    B = np.vectorize(code.get)(Bi).astype(np.uint8)
    sfa = np.ones((M, K // 128), np.float32)
    sfb = np.ones(((N + 127) // 128, K // 128), np.float32)
    expect = (Ai @ Bi.T).astype(np.float64)
    assert np.abs(expect).max() <= 256
    D = fg.fp8_gemm_nt(torch.from_numpy(A).cuda(), fg.get_col_major_tma_aligned_tensor(torch.from_numpy(sfa).cuda()),
                       torch.from_numpy(B).cuda(), torch.from_numpy(sfb).cuda())
    assert torch.equal(D.cpu().view(torch.int16), bf16_of(expect).view(torch.int16))


def test_repeated_launches_on_a_side_stream(fg):
    x = synth.normal_inputs(256, 512, 1024, seed=synth.seed_for(0, 70))
    A, sfa, B, sfb = to_gpu_normal(fg, x)
    s = torch.cuda.Stream()
    outs = []
    with torch.cuda.stream(s):
        for _ in range(3):
            outs.append(fg.fp8_gemm_nt(A, sfa, B, sfb))
    s.synchronize()
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    ref = oracle.gemm_nt(x.A.numpy(), x.sfa.numpy(), x.B.numpy(), x.sfb.numpy())
    check(outs[0].double().cpu().numpy(), ref)


@pytest.mark.parametrize("pair,bn,sms,M,N,K", [(0, 128, 8, 640, 640, 2048), (0, 128, 7, 640, 640, 2048),
                                               (0, 256, 9, 1024, 1280, 3072), (1, 256, 12, 1024, 1280, 3072),
                                               (1, 128, 12, 768, 640, 1536), (0, 64, 5, 384, 448, 1024)])
def test_stream_k_split_tiles_match_oracle(fg, monkeypatch, pair, bn, sms, M, N, K):
    """With the SM budget chosen so that the last wave of tiles is poorly
    filled, the tile kernel processes the first waves whole and splits the
    (tile, K block) iterations of the rest over the CTAs: pieces that end
    inside a tile publish FP32 partial sums, the piece that finishes a tile
    adds them in a fixed order.  Every element is checked against the oracle,
    and two launches must agree bit for bit."""
    monkeypatch.setenv("FG_FORCE_BLOCK_N", str(bn))
    monkeypatch.setenv("FG_FORCE_PAIR", str(pair))
    x = synth.normal_inputs(M, N, K, seed=synth.seed_for(0, 80) + bn + sms)
    A, sfa, B, sfb = to_gpu_normal(fg, x)
    full = fg.get_num_sms()
    try:
        fg.set_num_sms(sms)
        D1 = fg.fp8_gemm_nt(A, sfa, B, sfb)
        D2 = fg.fp8_gemm_nt(A, sfa, B, sfb)
        monkeypatch.setenv("FG_STREAMK", "0")
        D3 = fg.fp8_gemm_nt(A, sfa, B, sfb)
    finally:
        fg.set_num_sms(full)
    torch.cuda.synchronize()
    assert torch.equal(D1, D2)
    ref = oracle.gemm_nt(x.A.numpy(), x.sfa.numpy(), x.B.numpy(), x.sfb.numpy())
    check(D1.double().cpu().numpy(), ref)
    check(D3.double().cpu().numpy(), ref)


@pytest.mark.parametrize("pair", ["0", "1"])
def test_num_sms_limit_keeps_results(fg, pair, monkeypatch):
    """An SM budget changes only the schedule.  Without K splitting every
    output sums its K blocks in order, so the bits do not change; with 7 SMs
    the ragged last wave is split by stream-K, which regroups the FP32 sums
    (still deterministic, and within tolerance of the oracle).  The tile shape
    is fixed: tiles of another width or CTA pairing may round differently
    inside the tensor core."""
    monkeypatch.setenv("FG_FORCE_BLOCK_N", "128")
    monkeypatch.setenv("FG_FORCE_PAIR", pair)
    x = synth.normal_inputs(512, 1024, 512, seed=synth.seed_for(0, 71))
    A, sfa, B, sfb = to_gpu_normal(fg, x)
    ref = oracle.gemm_nt(x.A.numpy(), x.sfa.numpy(), x.B.numpy(), x.sfb.numpy())
    full = fg.get_num_sms()
    D0 = fg.fp8_gemm_nt(A, sfa, B, sfb)
    try:
        fg.set_num_sms(7)
        assert fg.get_num_sms() == 7
        D1 = fg.fp8_gemm_nt(A, sfa, B, sfb)
        D2 = fg.fp8_gemm_nt(A, sfa, B, sfb)
        monkeypatch.setenv("FG_STREAMK", "0")
        D3 = fg.fp8_gemm_nt(A, sfa, B, sfb)
    finally:
        fg.set_num_sms(full)
    torch.cuda.synchronize()
    assert torch.equal(D1, D2)
    assert torch.equal(D0, D3)
    check(D1.double().cpu().numpy(), ref)
    check(D0.double().cpu().numpy(), ref)


# ----------------------------------------------------------- grouped GEMMs --

def run_contiguous(fg, x):
    A = x.A.cuda()
    sfa = fg.get_col_major_tma_aligned_tensor(x.sfa.cuda())
    D = torch.full((x.M_tot, x.N), SENTINEL, dtype=torch.bfloat16, device="cuda")
    fg.m_grouped_fp8_gemm_nt_contiguous(A, sfa, x.B.cuda(), x.sfb.cuda(), x.m_indices.cuda(), D=D)
    torch.cuda.synchronize()
    return D


def check_contiguous(fg, x, D, rows=None):
    mi = x.m_indices.numpy()
    pad = mi < 0
    Dc = D.cpu()
    assert torch.all(Dc[torch.from_numpy(pad)].view(torch.int16) == sentinel_bf16().view(torch.int16))
    if rows is None:
        rows = np.nonzero(~pad)[0]
    ref, written = oracle.m_grouped_contiguous(x.A.numpy(), x.sfa.numpy(), x.B.numpy(), x.sfb.numpy(), mi,
                                               rows=rows)
    assert written.all()
    check(Dc[torch.from_numpy(np.asarray(rows))].double().numpy(), ref)


@pytest.mark.parametrize("pair", ["0", "1"])
def test_contiguous_small(fg, pair, monkeypatch):
    monkeypatch.setenv("FG_FORCE_PAIR", pair)
    x = synth.contiguous_inputs(4, 272, 512, seed=synth.seed_for(2, 50), counts=[5, 0, 130, 256])
    D = run_contiguous(fg, x)
    check_contiguous(fg, x, D)


@pytest.mark.parametrize("pair", ["0", "1"])
def test_contiguous_all_padding_block_is_skipped(fg, pair, monkeypatch):
    monkeypatch.setenv("FG_FORCE_PAIR", pair)
    x = synth.contiguous_inputs(2, 128, 256, seed=synth.seed_for(2, 51), counts=[100, 40])
    # add an all-padding block between the experts
    mi = x.m_indices.numpy()
    A = torch.cat([x.A[:128], torch.zeros((128, 256), dtype=torch.uint8), x.A[128:]])
    sfa = torch.cat([x.sfa[:128], torch.ones((128, 2)), x.sfa[128:]])
    tags = np.concatenate([mi[:128], np.full(128, -1, np.int32), mi[128:]])
    y = synth.ContiguousInputs(A, sfa, x.B, x.sfb, torch.from_numpy(tags), x.counts, 2, 128, 256)
    D = run_contiguous(fg, y)
    check_contiguous(fg, y, D)


def run_masked(fg, x, expected_m=0):
    sfa = fg.get_col_major_tma_aligned_tensor(x.sfa.cuda())
    D = torch.full((x.G, x.M_max, x.N), SENTINEL, dtype=torch.bfloat16, device="cuda")
    fg.m_grouped_fp8_gemm_nt_masked(x.A.cuda(), sfa, x.B.cuda(), x.sfb.cuda(), x.masked_m.cuda(),
                                    expected_m=expected_m, D=D)
    torch.cuda.synchronize()
    return D


def check_masked(fg, x, D, sample=None):
    mm = x.masked_m.numpy()
    Dc = D.cpu()
    lim = np.minimum(np.maximum(mm, 0), x.M_max)
    written = np.arange(x.M_max)[None, :] < lim[:, None]
    flat = Dc.view(-1, x.N)
    unw = torch.from_numpy(~written.reshape(-1))
    assert torch.all(flat[unw].view(torch.int16) == sentinel_bf16().view(torch.int16))
    rows = np.nonzero(written.reshape(-1))[0]
    if sample is not None and len(rows) > sample:
        rng = np.random.default_rng(0)
        rows = np.sort(rng.choice(rows, sample, replace=False))
    if len(rows) == 0:
        return
    ref, w = oracle.m_grouped_masked(x.A.numpy(), x.sfa.numpy(), x.B.numpy(), x.sfb.numpy(), mm, rows=rows)
    assert w.all()
    check(flat[torch.from_numpy(rows)].double().numpy(), ref)


@pytest.mark.parametrize("pair", ["0", "1"])
def test_masked_small(fg, pair, monkeypatch):
    monkeypatch.setenv("FG_FORCE_PAIR", pair)
    x = synth.masked_inputs(5, 200, 144, 384, seed=synth.seed_for(3, 50), masked=[0, 1, 128, 200, 250])
    D = run_masked(fg, x)
    check_masked(fg, x, D)


@pytest.mark.parametrize("pair", ["0", "1"])
def test_masked_all_empty(fg, pair, monkeypatch):
    monkeypatch.setenv("FG_FORCE_PAIR", pair)
    x = synth.masked_inputs(3, 64, 64, 128, seed=synth.seed_for(3, 51), masked=[0, 0, -5])
    D = run_masked(fg, x)
    check_masked(fg, x, D)


# ------------------------------------------- the workloads, at full size --

def sample_rows(M, n, seed):
    rng = np.random.default_rng(seed)
    rows = set([0, M - 1, min(M - 1, 127), min(M - 1, 128)])
    rows |= set(int(r) for r in rng.integers(0, M, n))
    return np.array(sorted(rows))


def block_edge_rows(M, n, seed):
    """The first and last row of every 128-row block (so every row tile of the
    kernel is checked on both sides of its boundaries) plus n random rows."""
    rows = set(sample_rows(M, n, seed).tolist())
    for b0 in range(0, M, 128):
        rows.add(b0)
        rows.add(min(M, b0 + 128) - 1)
    return np.array(sorted(rows))


def stratified_written_rows(written, labels, seed, per_segment=2):
    """Rows to check in a grouped output whose written rows form segments
    (runs of consecutive written rows with the same label: expert or group):
    the first and last written row of every segment, the written rows on
    either side of every 128-row block boundary inside it, and per_segment
    random rows of it."""
    rng = np.random.default_rng(seed)
    idx = np.nonzero(written)[0]
    if len(idx) == 0:
        return idx
    lab = np.asarray(labels)[idx]
    brk = (np.diff(idx) != 1) | (np.diff(lab) != 0)
    starts = np.concatenate([[0], np.nonzero(brk)[0] + 1])
    ends = np.concatenate([starts[1:], [len(idx)]])
    rows = set()
    for a, b in zip(starts, ends):
        seg = idx[a:b]
        rows |= {int(seg[0]), int(seg[-1])}
        rows |= set(int(r) for r in rng.choice(seg, min(per_segment, len(seg)), replace=False))
        for r in seg:
            if r % 128 == 0 or r % 128 == 127:
                rows.add(int(r))
    return np.array(sorted(rows))


def test_decode_config_full(fg):
    x = synth.normal_inputs(64, 2112, 7168, seed=synth.seed_for(0, 0))
    A, sfa, B, sfb = to_gpu_normal(fg, x)
    D = fg.fp8_gemm_nt(A, sfa, B, sfb)
    torch.cuda.synchronize()
    ref = oracle.gemm_nt(x.A.numpy(), x.sfa.numpy(), x.B.numpy(), x.sfb.numpy())
    check(D.double().cpu().numpy(), ref)


@pytest.mark.parametrize("si,N,K", [(0, 24576, 1536), (1, 7168, 16384), (2, 4096, 7168)])
def test_prefill_config_sampled_rows(fg, si, N, K):
    M = 4096
    x = synth.normal_inputs(M, N, K, seed=synth.seed_for(1, si))
    A, sfa, B, sfb = to_gpu_normal(fg, x)
    D = fg.fp8_gemm_nt(A, sfa, B, sfb)
    torch.cuda.synchronize()
    rows = block_edge_rows(M, 24, si)
    ref = oracle.gemm_nt(x.A.numpy(), x.sfa.numpy(), x.B.numpy(), x.sfb.numpy(), rows=rows)
    check(D[torch.from_numpy(rows).cuda()].double().cpu().numpy(), ref)


@pytest.mark.parametrize("si,N,K", [(0, 4096, 7168), (1, 7168, 2048)])
def test_contiguous_config_sampled_rows(fg, si, N, K):
    """Every expert is value-checked (first and last row, rows at each
    128-row block boundary, random rows), each against its own B and sfb."""
    x = synth.contiguous_inputs(8, N, K, seed=synth.seed_for(2, si))
    D = run_contiguous(fg, x)
    mi = x.m_indices.numpy()
    rows = stratified_written_rows(mi >= 0, mi, si)
    assert set(mi[rows].tolist()) == {e for e in range(8) if x.counts[e] > 0}
    Dc = D.cpu()
    assert torch.all(Dc[torch.from_numpy(mi < 0)].view(torch.int16) == sentinel_bf16().view(torch.int16))
    ref, written = oracle.m_grouped_contiguous(x.A.numpy(), x.sfa.numpy(), x.B.numpy(), x.sfb.numpy(), mi,
                                               rows=rows)
    assert written.all()
    got = Dc[torch.from_numpy(rows)].double().numpy()
    check(got, ref)
    for e in range(8):   # each expert's rows also meet the tolerance on their own
        sel = mi[rows] == e
        if sel.any():
            check(got[sel], ref[sel])


@pytest.mark.parametrize("si,N,K", [(0, 4096, 7168), (1, 7168, 2048)])
def test_masked_config_sampled_rows(fg, si, N, K):
    """Every non-empty group is value-checked (first and last row, rows at the
    128-row boundary, random rows), each against its own B and sfb."""
    x = synth.masked_inputs(32, 256, N, K, seed=synth.seed_for(3, si))
    D = run_masked(fg, x, expected_m=128)
    check_masked(fg, x, D, sample=0)
    mm = x.masked_m.numpy()
    lim = np.minimum(np.maximum(mm, 0), x.M_max)
    written = (np.arange(x.M_max)[None, :] < lim[:, None]).reshape(-1)
    rows = stratified_written_rows(written, np.arange(len(written)) // x.M_max, si)
    assert set((rows // x.M_max).tolist()) == {g for g in range(x.G) if lim[g] > 0}
    flat = D.view(-1, x.N)
    ref, w = oracle.m_grouped_masked(x.A.numpy(), x.sfa.numpy(), x.B.numpy(), x.sfb.numpy(), mm, rows=rows)
    assert w.all()
    check(flat[torch.from_numpy(rows).cuda()].double().cpu().numpy(), ref)
    for g in range(x.G):   # each group also meets the tolerance on its own
        sel = (rows // x.M_max) == g
        if sel.any():
            check(flat[torch.from_numpy(rows[sel]).cuda()].double().cpu().numpy(), ref[sel])


@pytest.mark.parametrize("si,M,N,K", [(i * 2 + j, M, N, K) for j, M in enumerate([64, 128])
                                      for i, (N, K) in enumerate([(2112, 7168), (24576, 1536), (32768, 512),
                                                                  (7168, 16384), (4096, 7168), (7168, 2048)])])
def test_decode_sweep_sampled_rows(fg, si, M, N, K):
    x = synth.normal_inputs(M, N, K, seed=synth.seed_for(4, si))
    A, sfa, B, sfb = to_gpu_normal(fg, x)
    D = fg.fp8_gemm_nt(A, sfa, B, sfb)
    torch.cuda.synchronize()
    rows = sample_rows(M, 8, si)
    ref = oracle.gemm_nt(x.A.numpy(), x.sfa.numpy(), x.B.numpy(), x.sfb.numpy(), rows=rows)
    check(D[torch.from_numpy(rows).cuda()].double().cpu().numpy(), ref)


# ------------------------------------------------------------ decode kernel --

@pytest.mark.parametrize("splits,reduce", [("1", "any"), ("3", "cluster"), ("3", "workspace"),
                                           ("5", "cluster"), ("5", "workspace"),
                                           ("8", "cluster"), ("8", "workspace")])
@pytest.mark.parametrize("M", [1, 17, 32, 64, 96, 100, 128, 160, 200, 256])
def test_decode_kernel_matches_oracle(fg, M, splits, reduce, monkeypatch):
    """Few rows of A: weights on the tensor core's 128-row side, K split over
    CTAs and reduced in split order, inside a cluster through distributed
    shared memory or through the global workspace; every token-tile width
    32..256.  Five splits of 8 K blocks leave the last split empty."""
    monkeypatch.setenv("FG_DECODE_MAX_M", "256")
    monkeypatch.setenv("FG_TILE_SPLITK", "0")
    monkeypatch.setenv("FG_FORCE_SPLITS", splits)
    monkeypatch.setenv("FG_DECODE_CLUSTER", "0" if reduce == "workspace" else "1")
    N, K = 400, 1024
    x = synth.normal_inputs(M, N, K, seed=synth.seed_for(4, 50) + M)
    A, sfa, B, sfb = to_gpu_normal(fg, x)
    D = fg.fp8_gemm_nt(A, sfa, B, sfb)
    torch.cuda.synchronize()
    ref = oracle.gemm_nt(x.A.numpy(), x.sfa.numpy(), x.B.numpy(), x.sfb.numpy())
    check(D.double().cpu().numpy(), ref)


def test_decode_repeated_and_interleaved_launches(fg, monkeypatch):
    """Split-K counters carry a launch epoch: back-to-back launches of
    different shapes on one stream must each reduce correctly."""
    monkeypatch.setenv("FG_FORCE_SPLITS", "5")
    xs = [synth.normal_inputs(64, 2112, 1280, seed=synth.seed_for(4, 60)),
          synth.normal_inputs(48, 1024, 2560, seed=synth.seed_for(4, 61))]
    dev = [to_gpu_normal(fg, x) for x in xs]
    outs = []
    for _ in range(3):
        for (A, sfa, B, sfb) in dev:
            outs.append(fg.fp8_gemm_nt(A, sfa, B, sfb))
    torch.cuda.synchronize()
    refs = [oracle.gemm_nt(x.A.numpy(), x.sfa.numpy(), x.B.numpy(), x.sfb.numpy()) for x in xs]
    for i, o in enumerate(outs):
        check(o.double().cpu().numpy(), refs[i % 2])
        assert torch.equal(o, outs[i % 2])   # deterministic reduction order


def test_decode_more_splits_than_a_cluster(fg, monkeypatch):
    """Above 8 splits the reduction always goes through the global workspace."""
    monkeypatch.setenv("FG_FORCE_SPLITS", "12")
    x = synth.normal_inputs(40, 528, 3072, seed=synth.seed_for(4, 64))
    A, sfa, B, sfb = to_gpu_normal(fg, x)
    D = fg.fp8_gemm_nt(A, sfa, B, sfb)
    torch.cuda.synchronize()
    ref = oracle.gemm_nt(x.A.numpy(), x.sfa.numpy(), x.B.numpy(), x.sfb.numpy())
    check(D.double().cpu().numpy(), ref)


@pytest.mark.parametrize("M,N,K,splits", [(64, 2112, 7168, "8"), (128, 4096, 7168, "4"), (5, 768, 2048, "2")])
def test_decode_cluster_and_workspace_reductions_agree(fg, M, N, K, splits, monkeypatch):
    """Both split-K reductions add the splits in the same order, so their
    results are equal element for element."""
    monkeypatch.setenv("FG_FORCE_SPLITS", splits)
    monkeypatch.setenv("FG_TILE_SPLITK", "0")
    x = synth.normal_inputs(M, N, K, seed=synth.seed_for(4, 63) + M)
    A, sfa, B, sfb = to_gpu_normal(fg, x)
    monkeypatch.setenv("FG_DECODE_CLUSTER", "1")
    D1 = fg.fp8_gemm_nt(A, sfa, B, sfb)
    monkeypatch.setenv("FG_DECODE_CLUSTER", "0")
    D2 = fg.fp8_gemm_nt(A, sfa, B, sfb)
    torch.cuda.synchronize()
    assert torch.equal(D1, D2)
    rows = sample_rows(M, 8, M)
    ref = oracle.gemm_nt(x.A.numpy(), x.sfa.numpy(), x.B.numpy(), x.sfb.numpy(), rows=rows)
    check(D1[torch.from_numpy(rows).cuda()].double().cpu().numpy(), ref)


@pytest.mark.parametrize("M,N,K", [(128, 4096, 7168), (100, 2112, 7168), (96, 7168, 2048), (65, 400, 1536),
                                   (1, 272, 1024), (17, 528, 640), (128, 256, 256), (128, 32768, 512)])
def test_tile_split_k_matches_oracle(fg, M, N, K, monkeypatch):
    """Few rows on the 128-row tile kernel with K split over the CTAs of a
    cluster and the partials summed through distributed shared memory in split
    order: every element against the oracle, ragged N and M, and the same
    bits on a second launch."""
    monkeypatch.setenv("FG_TILE_SPLITK", "1")
    plan = fg.query_plan("normal", M, N, K)
    tiles = -(-N // 256)
    if plan["kernel"] != "tile":
        pytest.skip(f"no resident cluster split for {tiles} tiles on this device: {plan}")
    assert plan["splits"] >= 2 and plan["cluster"] == plan["splits"]
    x = synth.normal_inputs(M, N, K, seed=synth.seed_for(4, 70) + M + N)
    A, sfa, B, sfb = to_gpu_normal(fg, x)
    D = torch.full((M, N), SENTINEL, dtype=torch.bfloat16, device="cuda")
    fg.fp8_gemm_nt(A, sfa, B, sfb, D=D)
    D2 = fg.fp8_gemm_nt(A, sfa, B, sfb)
    torch.cuda.synchronize()
    assert fg.get_last_device_status()[0] == 0
    assert torch.equal(D, D2)
    ref = oracle.gemm_nt(x.A.numpy(), x.sfa.numpy(), x.B.numpy(), x.sfb.numpy())
    check(D.double().cpu().numpy(), ref)


def test_tile_split_k_is_the_default_for_long_k_between_64_and_128_rows(fg, monkeypatch):
    monkeypatch.delenv("FG_TILE_SPLITK", raising=False)
    assert fg.query_plan("normal", 128, 7168, 16384)["kernel"] == "tile"
    assert fg.query_plan("normal", 64, 7168, 16384)["kernel"] == "decode"
    assert fg.query_plan("normal", 128, 7168, 2048)["kernel"] == "tile"
    plan = fg.query_plan("normal", 128, 4096, 7168)
    assert plan["kernel"] == "tile" and plan["tile_n"] == 128 and plan["splits"] >= 2


@pytest.mark.parametrize("M,N,K", [(128, 4096, 7168), (100, 4112, 7168), (77, 7184, 2048)])
def test_tile_split_k_128_wide_tiles_match_oracle(fg, M, N, K, monkeypatch):
    """The default plan for few rows and moderate K: 128-wide tiles (four TMEM
    accumulators), K split over a cluster, ragged M and a ragged last column
    block; every element against the oracle."""
    monkeypatch.delenv("FG_TILE_SPLITK", raising=False)
    monkeypatch.delenv("FG_FORCE_BLOCK_N", raising=False)
    plan = fg.query_plan("normal", M, N, K)
    assert plan["kernel"] == "tile" and plan["tile_n"] == 128 and plan["splits"] >= 2, plan
    x = synth.normal_inputs(M, N, K, seed=synth.seed_for(4, 71) + M)
    A, sfa, B, sfb = to_gpu_normal(fg, x)
    D = fg.fp8_gemm_nt(A, sfa, B, sfb)
    torch.cuda.synchronize()
    assert fg.get_last_device_status()[0] == 0
    ref = oracle.gemm_nt(x.A.numpy(), x.sfa.numpy(), x.B.numpy(), x.sfb.numpy())
    check(D.double().cpu().numpy(), ref)


def test_small_m_on_the_tile_kernel(fg, monkeypatch):
    """The 128-row tile kernel still handles few rows when the decode kernel is off."""
    monkeypatch.setenv("FG_DECODE_MAX_M", "0")
    x = synth.normal_inputs(64, 2112, 1024, seed=synth.seed_for(4, 62))
    A, sfa, B, sfb = to_gpu_normal(fg, x)
    D = fg.fp8_gemm_nt(A, sfa, B, sfb)
    torch.cuda.synchronize()
    ref = oracle.gemm_nt(x.A.numpy(), x.sfa.numpy(), x.B.numpy(), x.sfb.numpy())
    check(D.double().cpu().numpy(), ref)


# ------------------------------------------------------ failure detection --

FG_ERR_TIMEOUT = 6


@pytest.mark.parametrize("M,N,K,env,sms", [(4096, 4096, 7168, {}, 0),
                                           (64, 2112, 7168, {"FG_DECODE_CLUSTER": "0", "FG_FORCE_SPLITS": "8"}, 1)])
def test_wait_timeout_is_reported_and_the_context_stays_usable(fg, monkeypatch, M, N, K, env, sms):
    """With a 1 us limit on every pipeline wait, some wait of the GEMM runs
    out: the kernel records FG_ERR_TIMEOUT, stops its roles, drains its
    copies and returns.  The context must stay usable and the next call, with
    the normal limit, must be correct (split-K counters left behind by the
    abort are cleared when the status is read).  The decode case runs on one
    SM, so that its MMA issuers wait for whole split-K epilogues and several
    units pass through one CTA after the abort."""
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    x = synth.normal_inputs(M, N, K, seed=synth.seed_for(4, 70) + M)
    A, sfa, B, sfb = to_gpu_normal(fg, x)
    old = fg.get_wait_limit_ns()
    old_sms = fg.get_num_sms()
    codes = []
    try:
        if sms:
            fg.set_num_sms(sms)
        fg.set_wait_limit_ns(1000)
        for _ in range(5):
            fg.fp8_gemm_nt(A, sfa, B, sfb)
            codes.append(fg.get_last_device_status()[0])
            if codes[-1] == FG_ERR_TIMEOUT:
                break
    finally:
        fg.set_wait_limit_ns(old)
        fg.set_num_sms(old_sms)
    assert FG_ERR_TIMEOUT in codes, codes
    assert set(codes) <= {0, FG_ERR_TIMEOUT}
    D = fg.fp8_gemm_nt(A, sfa, B, sfb)
    torch.cuda.synchronize()
    assert fg.get_last_device_status()[0] == 0
    rows = sample_rows(M, 8, 70)
    ref = oracle.gemm_nt(x.A.numpy(), x.sfa.numpy(), x.B.numpy(), x.sfb.numpy(), rows=rows)
    check(D[torch.from_numpy(rows).cuda()].double().cpu().numpy(), ref)
