"""Failure detection without a GPU fault: the bounded waits.

Every mbarrier wait in the tensor-core kernels gives up after about one
second, records the timeout in the device error word and lets every warp of
the CTA leave, free its tensor memory and exit.  armt_test_bounded_wait runs
the grouped GEMM with its copy producer told to issue nothing, so the wait
for the first pipeline stage cannot complete (a flag that nothing sets).  The
test checks the status the host reads back, that the kernel ended within a
few seconds, and that the same process then computes normally (tensor memory
was released; the context is intact).
"""
import time

import numpy as np
import pytest

from .gpu_util import rel_l2

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_stays_usable():
    import torch
    from recurrent_memory_transformer_diag_b200 import grouped_gemm
    from recurrent_memory_transformer_diag_b200.armt import STATUS, lib
    st = torch.cuda.current_stream().cuda_stream
    for _ in range(2):   # twice: the first exit left nothing behind
        t0 = time.time()
        status = lib().armt_test_bounded_wait(st)
        dt = time.time() - t0
        assert STATUS[status] == "ARMT_ERR_DEVICE_TIMEOUT", STATUS.get(status, status)
        assert dt < 10.0, dt
    # a normal tensor-core product afterwards
    g = torch.Generator().manual_seed(3)
    A = torch.randn(2, 256, 512, generator=g).to(torch.bfloat16)
    B = (torch.randn(2, 256, 512, generator=g) * 0.05).to(torch.bfloat16)
    C = torch.empty(2, 256, 256, device="cuda")
    grouped_gemm(A.cuda(), B.cuda(), [1, 0], C)
    torch.cuda.synchronize()
    for i, b in enumerate([1, 0]):
        ref = A[i].double().numpy() @ B[b].double().numpy().T
        assert rel_l2(C[i].cpu().numpy(), ref) < 1e-5


def test_forward_after_timeout_is_clean():
    """A forward run after the timeout hook gives the same result as one run
    before it, and its own status word is clean."""
    import torch
    from recurrent_memory_transformer_diag_b200.armt import lib
    from recurrent_memory_transformer_diag_b200.inputs import CONFIGS, make_embeddings, make_weights
    from .gpu_util import run_gpu
    cfg = CONFIGS["small"]
    w = make_weights(cfg)
    emb = make_embeddings(cfg, 4)
    before = run_gpu(cfg, w, emb, 4)
    lib().armt_test_bounded_wait(torch.cuda.current_stream().cuda_stream)
    after = run_gpu(cfg, w, emb, 4)     # run_gpu checks armt_device_status
    for x, y in zip(before, after):
        np.testing.assert_array_equal(x, y)
