"""Single kernels through the unit entry points, against the oracle."""
import numpy as np
import pytest

import oracle

from .gpu_util import rel_l2

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("G,m,n,k,num_b", [
    (1, 128, 256, 64, 1),       # one tile, one k block
    (3, 1040, 512, 2048, 5),    # ragged M (8 full tiles + 16 rows), many k blocks
    (2, 144, 768, 688, 4),      # ragged K (10.75 k blocks)
    (4, 200, 64, 384, 2),       # N = 64 tile width
    (2, 77, 128, 136, 3),       # N = 128, tiny ragged M and K
    (16, 1040, 3072, 2048, 16), # a full 1B wave of QKV shapes
    (2, 512, 256, 128, 2),      # rows in whole 256-row CTA-pair tiles only
    (1, 300, 304, 200, 1),      # one pair tile + a 44-row one-CTA rest, ragged N and K
    # transposed ragged row tile (last tile of <= 16 rows, N a multiple of 128):
    (2, 144, 128, 256, 2),      # N = 128 tile, 16-row tail
    (1, 129, 256, 128, 1),      # a 1-row tail
    (2, 16, 256, 64, 1),        # a node of exactly 16 rows: its only tile transposed
    (3, 16, 2128, 2048, 3),     # the gated memory-write projection: 16 rows, N = 64 + 2048 + 16
    (40, 12, 2048, 128, 7),     # several transposed tiles per CTA (staging area reused)
    (2, 150, 256, 256, 2),      # a 22-row tail: an ordinary (partly filled) row tile
])
def test_tc_grouped_gemm_matches_fp64(G, m, n, k, num_b, dtype):
    import torch
    from recurrent_memory_transformer_diag_b200 import grouped_gemm
    g = torch.Generator().manual_seed(G * 1000 + m + n + k)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    A = torch.randn(G, m, k, generator=g).to(tdt)
    B = (torch.randn(num_b, n, k, generator=g) * 0.05).to(tdt)
    bidx = [(3 * i + 1) % num_b for i in range(G)]
    C = torch.full((G, m, n), float("nan"), device="cuda")
    grouped_gemm(A.cuda(), B.cuda(), bidx, C)
    torch.cuda.synchronize()
    got = C.cpu().numpy()
    An = A.float().numpy().astype(np.float64)
    Bn = B.float().numpy().astype(np.float64)
    for i in range(G):
        ref = An[i] @ Bn[bidx[i]].T
        assert rel_l2(got[i], ref) < 1e-5, (i, rel_l2(got[i], ref))


def test_simt_grouped_gemm_fp32_matches_fp64():
    import torch
    from recurrent_memory_transformer_diag_b200 import grouped_gemm
    g = torch.Generator().manual_seed(5)
    A = torch.randn(3, 70, 172, generator=g)
    B = torch.randn(2, 90, 172, generator=g)
    C = torch.empty(3, 70, 90, device="cuda")
    grouped_gemm(A.cuda(), B.cuda(), [1, 0, 1], C)
    torch.cuda.synchronize()
    for i, b in enumerate([1, 0, 1]):
        ref = A[i].double().numpy() @ B[b].double().numpy().T
        assert rel_l2(C[i].cpu().numpy(), ref) < 1e-6


# P = 2 dk nu: multiples of 4 take the 16-byte update kernel (P = 64, 384, 768;
# M = 32 the widest lane map; M = 5 an odd count before the prefetch ring),
# P = 10 and 42 the scalar one
@pytest.mark.parametrize("M,d,dk,nu", [(4, 64, 16, 2), (16, 256, 64, 3), (16, 2048, 64, 3), (16, 3072, 128, 3),
                                       (32, 128, 16, 2), (3, 64, 5, 1), (16, 96, 7, 3), (5, 64, 8, 2)])
def test_memory_write_matches_oracle(M, d, dk, nu):
    import torch
    from recurrent_memory_transformer_diag_b200 import memory_write
    rng = np.random.default_rng(M + d)
    P = 2 * dk * nu
    m = rng.standard_normal((M, d)).astype(np.float32)
    wk = (0.02 * rng.standard_normal((dk, d))).astype(np.float32)
    wv = (0.02 * rng.standard_normal((d, d))).astype(np.float32)
    # a non-trivial prior state: two earlier writes
    A0 = np.zeros((d, P))
    z0 = np.zeros(P)
    for _ in range(2):
        prev = rng.standard_normal((M, d)).astype(np.float32)
        A0, z0 = oracle.mem_write(prev, wk, wv, A0, z0, nu, 1e-5)
    A0 = A0.astype(np.float32)
    z0 = z0.astype(np.float32)
    Ar, zr = oracle.mem_write(m, wk, wv, A0, z0, nu, 1e-5)
    At = torch.from_numpy(A0).cuda()
    zt = torch.from_numpy(z0).cuda()
    memory_write(torch.from_numpy(m).cuda(), torch.from_numpy(wk).cuda(), torch.from_numpy(wv).cuda(),
                 At, zt, nu, 1e-5)
    torch.cuda.synchronize()
    assert rel_l2(At.cpu().numpy(), Ar) < 1e-5
    assert rel_l2(zt.cpu().numpy(), zr) < 1e-5


@pytest.mark.parametrize("G,m,n,k,num_b", [
    (2, 1040, 2048, 384, 16),   # the memory-read product at the 1B shape (K = P)
    (3, 144, 256, 96, 2),       # ragged M, K of 3 k-blocks of 32 words
    (2, 77, 64, 40, 1),         # N = 64 tile, ragged K (1.25 k-blocks)
    (1, 300, 128, 768, 1),      # N = 128, the 3B P
    (2, 10, 128, 96, 1),        # N = 128, a 10-row node (transposed tile)
])
def test_tc_grouped_gemm_tf32_matches_fp64(G, m, n, k, num_b):
    """fp32 operands on kind::tf32: each operand enters at tf32 precision
    (10-bit mantissa, relative error <= 2^-10 per operand whether rounded or
    truncated), so a product term is within ~2^-9 and the rel-L2 of the sum of
    random-sign terms stays well below 2e-3."""
    import torch
    from recurrent_memory_transformer_diag_b200 import grouped_gemm
    g = torch.Generator().manual_seed(G * 7 + m + n + k)
    A = torch.randn(G, m, k, generator=g)
    B = torch.randn(num_b, n, k, generator=g) * 0.05
    bidx = [(2 * i + 1) % num_b for i in range(G)]
    C = torch.full((G, m, n), float("nan"), device="cuda")
    grouped_gemm(A.cuda(), B.cuda(), bidx, C, tf32=True)
    torch.cuda.synchronize()
    got = C.cpu().numpy()
    for i in range(G):
        ref = A[i].double().numpy() @ B[bidx[i]].double().numpy().T
        err = rel_l2(got[i], ref)
        assert 0 < err < 2e-3, (i, err)     # > 0: the product really ran at reduced precision


SWAP_OFF_CHILD = """
import numpy as np, torch
from recurrent_memory_transformer_diag_b200 import grouped_gemm
for G, m, n, k, num_b, tf32 in [(3, 1040, 512, 2048, 5, False), (3, 16, 2128, 2048, 3, False),
                                (2, 1040, 2048, 384, 16, True)]:
    g = torch.Generator().manual_seed(G * 1000 + m + n + k)
    A = torch.randn(G, m, k, generator=g)
    B = torch.randn(num_b, n, k, generator=g) * 0.05
    if not tf32:
        A, B = A.to(torch.bfloat16), B.to(torch.bfloat16)
    bidx = [(3 * i + 1) % num_b for i in range(G)]
    C = torch.full((G, m, n), float("nan"), device="cuda")
    grouped_gemm(A.cuda(), B.cuda(), bidx, C, tf32=tf32)
    torch.cuda.synchronize()
    got = C.cpu().double().numpy()
    An = A.double().numpy(); Bn = B.double().numpy()
    for i in range(G):
        ref = An[i] @ Bn[bidx[i]].T
        err = np.linalg.norm(got[i] - ref) / np.linalg.norm(ref)
        assert err < (2e-3 if tf32 else 1e-5), (G, m, n, k, i, err)
print("SWAP_OFF_OK")
"""


def test_tc_grouped_gemm_without_transposed_tail():
    """ARMT_GEMM_SWAP_TAIL=0 (the A/B switch) keeps the ragged last row tile
    on the ordinary 128-row product; both layouts match the fp64 product."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, ARMT_GEMM_SWAP_TAIL="0")
    r = subprocess.run([sys.executable, "-c", SWAP_OFF_CHILD], cwd=root, env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "SWAP_OFF_OK" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
