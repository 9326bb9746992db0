"""Seeded synthetic inputs for the FP8 GEMM tests and benchmark.

This module holds none of the GEMM's arithmetic.  It draws N(0,1) fp32 values
from a seeded ``torch.Generator`` and turns them into E4M3 codes plus FP32 block
scales with torch's own ``float8_e4m3fn`` cast (a library routine), following
the recipe of the workloads: scale = max(amax, 1e-4) / 448 per 1x128 row block
of A and per 128x128 block of B, codes = cast(clamp(x / scale, -448, 448)).
Both the CUDA path and the CPU oracle consume the same bytes and scales, so how
they were made never affects parity.

Values are generated in row chunks of ``CHUNK_ROWS`` rows (a multiple of 128, so
no 128x128 block straddles two chunks); the CPU and CUDA generators give
different streams for the same seed, so a test that compares against the
oracle generates on the CPU and uploads.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

BLOCK = 128
CHUNK_ROWS = 2048
E4M3_MAX = 448.0
AMAX_FLOOR = 1e-4


def seed_for(config_index: int, shape_index: int = 0) -> int:
    """Seed of one workload shape: 20260000 + 100 * config + shape."""
    return 20260000 + 100 * config_index + shape_index


def _ceil_div(a: int, b: int) -> int:
    return (a + b - 1) // b


def _quantize_chunk(x: torch.Tensor, block_rows: int):
    """x [r, C] fp32 (r a multiple of block_rows unless it is the last chunk)
    -> (codes uint8 [r, C], scales fp32 [ceil(r/block_rows), ceil(C/128)])."""
    r, C = x.shape
    rp = _ceil_div(r, block_rows) * block_rows
    cp = _ceil_div(C, BLOCK) * BLOCK
    xp = x
    if rp != r or cp != C:
        xp = torch.zeros((rp, cp), dtype=x.dtype, device=x.device)
        xp[:r, :C] = x
    blocks = xp.view(rp // block_rows, block_rows, cp // BLOCK, BLOCK)
    amax = blocks.abs().amax(dim=(1, 3))
    scale = amax.clamp(min=AMAX_FLOOR) / E4M3_MAX
    q = (blocks / scale[:, None, :, None]).clamp(-E4M3_MAX, E4M3_MAX)
    q = q.to(torch.float8_e4m3fn).view(torch.uint8).reshape(rp, cp)[:r, :C]
    return q.contiguous(), scale.contiguous()


def randn_quantized(R: int, C: int, block_rows: int, gen: torch.Generator,
                    device="cpu"):
    """Draw x ~ N(0,1) [R, C] in chunks and quantise with block_rows x 128
    blocks.  Returns (codes uint8 [R, C], scales fp32 [ceil(R/br), ceil(C/128)])."""
    q = torch.empty((R, C), dtype=torch.uint8, device=device)
    s = torch.empty((_ceil_div(R, block_rows), _ceil_div(C, BLOCK)), dtype=torch.float32,
                    device=device)
    for r0 in range(0, R, CHUNK_ROWS):
        r1 = min(R, r0 + CHUNK_ROWS)
        x = torch.randn((r1 - r0, C), generator=gen, dtype=torch.float32, device=device)
        qc, sc = _quantize_chunk(x, block_rows)
        q[r0:r1] = qc
        s[r0 // block_rows: r0 // block_rows + sc.shape[0]] = sc
    return q, s


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


@dataclass
class NormalInputs:
    A: torch.Tensor        # uint8 [M, K] E4M3 codes
    sfa: torch.Tensor      # fp32 [M, K/128], row-major (one scale per 1x128 block)
    B: torch.Tensor        # uint8 [N, K]
    sfb: torch.Tensor      # fp32 [ceil(N/128), K/128]
    M: int
    N: int
    K: int


def normal_inputs(M: int, N: int, K: int, seed: int, device="cpu") -> NormalInputs:
    g = _gen(seed, device)
    A, sfa = randn_quantized(M, K, 1, g, device)
    B, sfb = randn_quantized(N, K, BLOCK, g, device)
    return NormalInputs(A, sfa, B, sfb, M, N, K)


@dataclass
class ContiguousInputs:
    A: torch.Tensor        # uint8 [M_tot, K]
    sfa: torch.Tensor      # fp32 [M_tot, K/128]
    B: torch.Tensor        # uint8 [G, N, K]
    sfb: torch.Tensor      # fp32 [G, ceil(N/128), K/128]
    m_indices: torch.Tensor  # int32 [M_tot], expert id or -1 on padding rows
    counts: list = field(default_factory=list)  # real rows per expert
    G: int = 0
    N: int = 0
    K: int = 0

    @property
    def M_tot(self) -> int:
        return self.A.shape[0]


def contiguous_counts(G: int, seed: int, lo: int = 1024, hi: int = 8192) -> list:
    """Rows per expert drawn uniformly from the integers [lo, hi]."""
    rng = np.random.default_rng(seed)
    return [int(v) for v in rng.integers(lo, hi, size=G, endpoint=True)]


def contiguous_inputs(G: int, N: int, K: int, seed: int, counts=None, align: int = BLOCK,
                      device="cpu") -> ContiguousInputs:
    """Expert segments of ``counts[e]`` rows, each padded with -1 rows up to a
    multiple of ``align`` and concatenated along M."""
    if counts is None:
        counts = contiguous_counts(G, seed)
    padded = [_ceil_div(c, align) * align for c in counts]
    M_tot = int(sum(padded))
    tags = np.full(M_tot, -1, dtype=np.int32)
    r = 0
    for e, (c, p) in enumerate(zip(counts, padded)):
        tags[r:r + c] = e
        r += p
    g = _gen(seed, device)
    A, sfa = randn_quantized(M_tot, K, 1, g, device)
    B = torch.empty((G, N, K), dtype=torch.uint8, device=device)
    sfb = torch.empty((G, _ceil_div(N, BLOCK), K // BLOCK), dtype=torch.float32, device=device)
    for e in range(G):
        B[e], sfb[e] = randn_quantized(N, K, BLOCK, g, device)
    m_indices = torch.from_numpy(tags).to(device)
    return ContiguousInputs(A, sfa, B, sfb, m_indices, list(counts), G, N, K)


@dataclass
class MaskedInputs:
    A: torch.Tensor        # uint8 [G, M_max, K]
    sfa: torch.Tensor      # fp32 [G, M_max, K/128]
    B: torch.Tensor        # uint8 [G, N, K]
    sfb: torch.Tensor      # fp32 [G, ceil(N/128), K/128]
    masked_m: torch.Tensor  # int32 [G]
    G: int = 0
    M_max: int = 0
    N: int = 0
    K: int = 0


def masked_counts(G: int, seed: int, lo: int = 0, hi: int = 256) -> list:
    rng = np.random.default_rng(seed)
    return [int(v) for v in rng.integers(lo, hi, size=G, endpoint=True)]


def masked_inputs(G: int, M_max: int, N: int, K: int, seed: int, masked=None,
                  device="cpu") -> MaskedInputs:
    if masked is None:
        masked = masked_counts(G, seed, 0, M_max)
    g = _gen(seed, device)
    A, sfa = randn_quantized(G * M_max, K, 1, g, device)
    B = torch.empty((G, N, K), dtype=torch.uint8, device=device)
    sfb = torch.empty((G, _ceil_div(N, BLOCK), K // BLOCK), dtype=torch.float32, device=device)
    for e in range(G):
        B[e], sfb[e] = randn_quantized(N, K, BLOCK, g, device)
    mm = torch.tensor(masked, dtype=torch.int32, device=device)
    return MaskedInputs(A.view(G, M_max, K), sfa.view(G, M_max, K // BLOCK), B, sfb, mm,
                        G, M_max, N, K)


def random_codes(shape, gen: torch.Generator, device="cpu", allow_nan: bool = False):
    """Uniform random E4M3 codes (NaN codes 0x7F/0xFF excluded unless allowed)."""
    c = torch.randint(0, 256, shape, generator=gen, dtype=torch.int32, device=device)
    if not allow_nan:
        c = torch.where((c & 0x7F) == 0x7F, c - 1, c)
    return c.to(torch.uint8)
