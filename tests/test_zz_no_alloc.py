"""armt_memory_write_static, the delta-rule memory write for callers that
cannot allocate device memory at call time (a framework that has reserved
the device memory for its own allocator, a real-time loop with a fixed
memory budget): it must give the same state as armt_memory_write, which
takes its scratch from cudaMallocAsync, on consecutive calls that share the
library's fixed scratch array.  Collected last so that a failure here comes
after every other test has run."""
import numpy as np
import pytest

from .gpu_util import rel_l2

pytestmark = pytest.mark.gpu


def _case(M, d, dk, nu, seed):
    rng = np.random.default_rng(seed)
    f = np.float32
    m1 = rng.standard_normal((M, d)).astype(f)
    m2 = rng.standard_normal((M, d)).astype(f)
    wk = (0.02 * rng.standard_normal((dk, d))).astype(f)
    wv = (0.02 * rng.standard_normal((d, d))).astype(f)
    P = 2 * dk * nu
    A0 = (1e-3 * rng.standard_normal((d, P))).astype(f)
    z0 = np.abs(rng.standard_normal(P)).astype(f)
    return m1, m2, wk, wv, A0, z0


# The last three shapes make M*(dk+d) (the projected rows that precede the
# DPFP features in the scratch) not a multiple of 4 floats, so the feature
# rows start only where the scratch layout pads them to 16 bytes.
@pytest.mark.parametrize("M,d,dk,nu", [(16, 2048, 64, 3), (4, 64, 16, 2), (16, 3072, 128, 3),
                                       (1, 64, 2, 1), (3, 65, 2, 2), (5, 130, 8, 2)])
def test_static_write_matches_allocating_write_on_two_calls(M, d, dk, nu):
    import torch
    from recurrent_memory_transformer_diag_b200 import memory_write, memory_write_static
    m1, m2, wk, wv, A0, z0 = _case(M, d, dk, nu, seed=M + d)
    dev = lambda x: torch.from_numpy(x).cuda()
    wk_d, wv_d = dev(wk), dev(wv)
    # reference: the allocating entry point, two writes in a row
    A_ref, z_ref = dev(A0), dev(z0)
    memory_write(dev(m1), wk_d, wv_d, A_ref, z_ref, nu, 1e-5)
    torch.cuda.synchronize()
    A_ref1, z_ref1 = A_ref.cpu().numpy(), z_ref.cpu().numpy()
    memory_write(dev(m2), wk_d, wv_d, A_ref, z_ref, nu, 1e-5)
    torch.cuda.synchronize()
    # the no-allocation entry point, the same two writes in a row
    A, z = dev(A0), dev(z0)
    memory_write_static(dev(m1), wk_d, wv_d, A, z, nu, 1e-5)
    torch.cuda.synchronize()
    assert rel_l2(A.cpu().numpy(), A_ref1) < 1e-5
    assert rel_l2(z.cpu().numpy(), z_ref1) < 1e-5
    memory_write_static(dev(m2), wk_d, wv_d, A, z, nu, 1e-5)
    torch.cuda.synchronize()
    assert rel_l2(A.cpu().numpy(), A_ref.cpu().numpy()) < 1e-5
    assert rel_l2(z.cpu().numpy(), z_ref.cpu().numpy()) < 1e-5


def _default_pool_used():
    """(current, high-water) bytes in use in the device's default memory pool,
    the pool cudaMallocAsync draws from."""
    import torch
    from cuda.bindings import runtime as rt
    err, pool = rt.cudaDeviceGetDefaultMemPool(torch.cuda.current_device())
    assert err == rt.cudaError_t.cudaSuccess
    out = []
    for attr in (rt.cudaMemPoolAttr.cudaMemPoolAttrUsedMemCurrent, rt.cudaMemPoolAttr.cudaMemPoolAttrUsedMemHigh):
        err, v = rt.cudaMemPoolGetAttribute(pool, attr)
        assert err == rt.cudaError_t.cudaSuccess
        out.append(int(v))
    return out


def _reset_pool_high_water():
    import torch
    from cuda.bindings import driver as dr, runtime as rt
    err, pool = rt.cudaDeviceGetDefaultMemPool(torch.cuda.current_device())
    assert err == rt.cudaError_t.cudaSuccess
    err, = rt.cudaMemPoolSetAttribute(pool, rt.cudaMemPoolAttr.cudaMemPoolAttrUsedMemHigh, dr.cuuint64_t(0))
    assert err == rt.cudaError_t.cudaSuccess


def test_static_write_takes_nothing_from_the_allocators():
    """Neither the stream-ordered pool nor torch's allocator grows during the
    no-allocation write, even transiently (the pool's high-water mark is reset
    first); the allocating write, run the same way, does raise the mark."""
    import torch
    from recurrent_memory_transformer_diag_b200 import memory_write, memory_write_static
    M, d, dk, nu = 16, 2048, 64, 3
    m1, m2, wk, wv, A0, z0 = _case(M, d, dk, nu, seed=7)
    dev = lambda x: torch.from_numpy(x).cuda()
    m1_d, m2_d, wk_d, wv_d, A, z = dev(m1), dev(m2), dev(wk), dev(wv), dev(A0), dev(z0)
    memory_write_static(m1_d, wk_d, wv_d, A, z, nu, 1e-5)   # first call on the device: set-up
    torch.cuda.synchronize()
    torch_before = torch.cuda.memory_allocated()
    _reset_pool_high_water()
    used0, _ = _default_pool_used()
    memory_write_static(m2_d, wk_d, wv_d, A, z, nu, 1e-5)
    memory_write_static(m1_d, wk_d, wv_d, A, z, nu, 1e-5)
    torch.cuda.synchronize()
    used1, high1 = _default_pool_used()
    assert used1 == used0 and high1 <= used0
    assert torch.cuda.memory_allocated() == torch_before
    # positive control: the check sees the allocating entry point's scratch
    _reset_pool_high_water()
    memory_write(m2_d, wk_d, wv_d, A, z, nu, 1e-5)
    torch.cuda.synchronize()
    _, high2 = _default_pool_used()
    assert high2 > used0


def test_static_write_rejects_sizes_beyond_its_scratch():
    import torch
    from recurrent_memory_transformer_diag_b200 import ArmtError, memory_write_static
    M, d, dk, nu = 32, 16384, 64, 3         # M*(dk+d) alone exceeds the 1 MiB array
    m = torch.zeros(M, d, device="cuda")
    wk = torch.zeros(dk, d, device="cuda")
    wv = torch.zeros(8, 8, device="cuda")   # never read: the call is rejected first
    A = torch.zeros(d, 2 * dk * nu, device="cuda")
    z = torch.zeros(2 * dk * nu, device="cuda")
    with pytest.raises(ArmtError) as ei:
        memory_write_static(m, wk, wv, A, z, nu, 1e-5)
    assert ei.value.name == "ARMT_ERR_SHAPE"
