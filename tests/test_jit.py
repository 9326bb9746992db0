"""Runtime specialisation of the tile kernel (FG_JIT=1): NVRTC compilation
with the K block count as a compile-time constant, and the on-disk cache that
later processes reuse.  The compilation needs no GPU; the GPU tests run a
GEMM through the runtime-compiled kernel in two fresh processes and check it
against the CPU oracle."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_compile_and_disk_cache(tmp_path, monkeypatch):
    import fp8_fine_grained_tma_b200 as fg
    monkeypatch.setenv("FG_CACHE_DIR", str(tmp_path))
    before = fg.jit_stats()
    p1 = fg.jit_compile(256, False, 56)
    assert os.path.exists(p1) and os.path.getsize(p1) > 10000
    mid = fg.jit_stats()
    assert mid["compiled"] == before["compiled"] + 1
    assert fg.jit_compile(256, False, 56) == p1            # the same specialisation comes from the cache
    assert fg.jit_stats()["loaded_from_disk"] == mid["loaded_from_disk"] + 1
    p2 = fg.jit_compile(256, False, 57)
    p3 = fg.jit_compile(128, True, 56)
    assert len({p1, p2, p3}) == 3                           # one cubin per specialisation
    for bad in [(8, False, 4), (256, False, 0), (16, True, 4), (300, False, 4)]:
        with pytest.raises(fg.FG8Error):
            fg.jit_compile(*bad)


CHILD = r"""
import json, sys
sys.path.insert(0, ROOT)
import numpy as np, torch
import fp8_fine_grained_tma_b200 as fg, oracle, synth
M, N, K = 512, 1024, 2048
x = synth.normal_inputs(M, N, K, seed=20261234)
sfa = fg.get_col_major_tma_aligned_tensor(x.sfa.cuda())
D = fg.fp8_gemm_nt(x.A.cuda(), sfa, x.B.cuda(), x.sfb.cuda())
torch.cuda.synchronize()
ref = oracle.gemm_nt(x.A.numpy(), x.sfa.numpy(), x.B.numpy(), x.sfb.numpy())
c = oracle.compare(D.double().cpu().numpy(), ref)
print(json.dumps({"stats": fg.jit_stats(), "diff": c["diff"], "rel": c["rel_max_err"],
                  "status": fg.get_last_device_status()[0]}))
"""


@pytest.mark.gpu
def test_runtime_compiled_kernel_matches_oracle_and_is_reused(tmp_path):
    env = dict(os.environ, FG_JIT="1", FG_CACHE_DIR=str(tmp_path / "cache"), FG_FORCE_BLOCK_N="128")
    code = "ROOT = %r\n" % ROOT + CHILD
    outs = []
    for _ in range(2):
        r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
        assert r.returncode == 0, r.stderr[-2000:]
        outs.append(json.loads(r.stdout.strip().splitlines()[-1]))
    first, second = outs
    assert first["stats"]["compiled"] == 1 and first["stats"]["launches"] >= 1
    assert second["stats"]["compiled"] == 0 and second["stats"]["loaded_from_disk"] == 1
    assert second["stats"]["launches"] >= 1
    for o in outs:
        assert o["status"] == 0
        assert o["diff"] <= 1e-3 and o["rel"] <= 1e-2, o
