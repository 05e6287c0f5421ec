"""The CTA-pair (cta_group::2) grouped GEMM, enabled through the environment
in a child process, against an fp64 product (the one-CTA kernel is the
default and is covered by test_kernels_gpu.py)."""
import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import numpy as np, torch
    from recurrent_memory_transformer_diag_b200 import grouped_gemm
    cases = [(2, 512, 256, 128, 2), (1, 300, 304, 200, 1), (3, 1040, 512, 2048, 5), (4, 1040, 3072, 2048, 4)]
    for G, m, n, k, num_b in cases:
        for tdt in (torch.bfloat16, torch.float16):
            g = torch.Generator().manual_seed(G * 1000 + m + n + k)
            A = torch.randn(G, m, k, generator=g).to(tdt)
            B = (torch.randn(num_b, n, k, generator=g) * 0.05).to(tdt)
            bidx = [(3 * i + 1) % num_b for i in range(G)]
            C = torch.full((G, m, n), float("nan"), device="cuda")
            grouped_gemm(A.cuda(), B.cuda(), bidx, C)
            torch.cuda.synchronize()
            got = C.cpu().double().numpy()
            An = A.double().numpy(); Bn = B.double().numpy()
            for i in range(G):
                ref = An[i] @ Bn[bidx[i]].T
                err = np.linalg.norm(got[i] - ref) / np.linalg.norm(ref)
                assert err < 1e-5, (G, m, n, k, i, err)
    print("PAIRS_OK")
""")


def test_cta_pair_gemm_matches_fp64():
    env = dict(os.environ, ARMT_GEMM_CTA_PAIRS="1")
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "PAIRS_OK" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
