"""GPU forward vs the fp64 oracle, through the C ABI.

Tolerances (relative L2 error, each output and each layer separately):
fp32 mode <= 1e-5, bf16 mode <= 1e-2 (the target the build states for the
two numeric modes).
"""
import numpy as np
import pytest

import oracle
from recurrent_memory_transformer_diag_b200.inputs import CONFIGS, make_embeddings, make_weights

from .gpu_util import rel_l2, run_gpu

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-5, "bf16": 1e-2}


def _compare(cfg, got, ref, tol):
    h, A, z = got
    hr, Ar, zr = ref
    assert np.isfinite(h).all() and np.isfinite(A).all() and np.isfinite(z).all()
    errs = {"hidden": rel_l2(h, hr)}
    T = cfg.seg_len
    for s in range(h.shape[0] // T):   # per segment: a wrong segment cannot hide under the average
        errs[f"hidden[seg {s}]"] = rel_l2(h[s * T:(s + 1) * T], hr[s * T:(s + 1) * T])
    for l in range(cfg.n_layers):
        errs[f"A[{l}]"] = rel_l2(A[l], Ar[l])
        errs[f"z[{l}]"] = rel_l2(z[l], zr[l])
    worst = max(errs, key=errs.get)
    print(f"\n{cfg.name}: rel-L2 hidden {errs['hidden']:.3e}, worst {worst} {errs[worst]:.3e} (tol {tol})")
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f"rel-L2 above {tol}: {bad}"
    return errs


@pytest.fixture(scope="module")
def tiny():
    cfg = CONFIGS["tiny"]
    w = make_weights(cfg)
    emb = make_embeddings(cfg)
    return cfg, w, emb, oracle.forward(cfg, w, emb)


@pytest.fixture(scope="module")
def small():
    cfg = CONFIGS["small"]
    w = make_weights(cfg)
    emb = make_embeddings(cfg)
    return cfg, w, emb, oracle.forward(cfg, w, emb)


@pytest.mark.parametrize("schedule", ["diagonal", "sequential"])
def test_tiny_fp32_matches_oracle(tiny, schedule):
    cfg, w, emb, ref = tiny
    got = run_gpu(cfg, w, emb, cfg.n_segments, schedule=schedule)
    _compare(cfg, got, ref, TOL["fp32"])


@pytest.mark.parametrize("schedule", ["diagonal", "sequential"])
def test_small_bf16_matches_oracle(small, schedule):
    cfg, w, emb, ref = small
    got = run_gpu(cfg, w, emb, cfg.n_segments, schedule=schedule)
    _compare(cfg, got, ref, TOL["bf16"])


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_diagonal_equals_sequential_bitwise(name):
    """Each node is computed by the same kernels on the same inputs in both
    schedules, so the outputs are bit-identical."""
    cfg = CONFIGS[name]
    w = make_weights(cfg)
    emb = make_embeddings(cfg)
    a = run_gpu(cfg, w, emb, cfg.n_segments, schedule="diagonal")
    b = run_gpu(cfg, w, emb, cfg.n_segments, schedule="sequential")
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_graph_and_direct_launch_agree_and_repeat(small):
    cfg, w, emb, _ = small
    a = run_gpu(cfg, w, emb, cfg.n_segments, graph=True, repeat=2)
    b = run_gpu(cfg, w, emb, cfg.n_segments, graph=False)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


@pytest.mark.parametrize("S", [1, 2, 5])
def test_small_ragged_segment_counts(small, S):
    """S below L (partial waves), S = 1 (no memory read), odd S."""
    cfg, w, emb, _ = small
    e = emb[:S * cfg.seg_len]
    ref = oracle.forward(cfg, w, e)
    got = run_gpu(cfg, w, e, S, max_segments=cfg.n_segments)
    _compare(cfg, got, ref, TOL["bf16"])


def test_small_short_segments(small):
    """seg_len below the maximum the context was created for (T' = 40 rows)."""
    cfg, w, _, _ = small
    c2 = cfg.with_(seg_len=24, n_segments=6)
    emb = make_embeddings(c2)
    ref = oracle.forward(c2, w, emb)
    import torch
    from recurrent_memory_transformer_diag_b200 import Armt
    m = Armt(cfg)
    m.load_weights(w)
    got = run_gpu(c2, w, emb, 6, model=m)
    m.close()
    _compare(c2, got, ref, TOL["bf16"])
    del torch


@pytest.mark.parametrize("pinned", [True, False])
def test_host_buffer_forward_matches_device_forward(small, pinned):
    """Page-locked buffers take the path whose per-segment copies overlap the
    waves (one graph over three streams, run twice to replay it); pageable ones
    the copy-forward-copy path.  Both must equal the device-buffer forward."""
    cfg, w, emb, _ = small
    import torch
    from recurrent_memory_transformer_diag_b200 import Armt
    dev = run_gpu(cfg, w, emb, cfg.n_segments)
    m = Armt(cfg)
    m.load_weights(w)
    S, T, L, d, P = cfg.n_segments, cfg.seg_len, cfg.n_layers, cfg.d_model, cfg.phi_dim
    pin = (lambda t: t.pin_memory()) if pinned else (lambda t: t)
    e = pin(torch.from_numpy(emb).to(torch.bfloat16))
    out = pin(torch.empty(S * T, d, dtype=torch.bfloat16))
    A = pin(torch.empty(L, d, P, dtype=torch.float32))
    z = pin(torch.empty(L, P, dtype=torch.float32))
    for _ in range(2):
        out.fill_(float("nan")); A.fill_(float("nan")); z.fill_(float("nan"))
        m.forward_host(e, S, T, out, A, z)
        np.testing.assert_array_equal(out.float().numpy(), dev[0])
        np.testing.assert_array_equal(A.numpy(), dev[1])
        np.testing.assert_array_equal(z.numpy(), dev[2])
    m.close()


def test_errors_through_the_abi(small):
    cfg, w, emb, _ = small
    import torch
    from recurrent_memory_transformer_diag_b200 import Armt, ArmtError
    m = Armt(cfg, max_segments=4)
    e = torch.zeros(4 * cfg.seg_len, cfg.d_model, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(e)
    A = torch.empty(cfg.n_layers, cfg.d_model, cfg.phi_dim, device="cuda")
    z = torch.empty(cfg.n_layers, cfg.phi_dim, device="cuda")
    with pytest.raises(ArmtError) as ei:
        m.forward(e, 4, cfg.seg_len, out, A, z)
    assert ei.value.name == "ARMT_ERR_NOT_LOADED"
    m.load_weights(w)
    with pytest.raises(ArmtError) as ei:
        m.forward(e, 5, cfg.seg_len, out, A, z)
    assert ei.value.name == "ARMT_ERR_SHAPE"
    with pytest.raises(ArmtError) as ei:
        m.forward(e, 4, cfg.seg_len + 1, out, A, z)
    assert ei.value.name == "ARMT_ERR_SHAPE"
    with pytest.raises(ArmtError) as ei:
        m.forward(e, 0, cfg.seg_len, out, A, z)
    assert ei.value.name == "ARMT_ERR_INVALID_ARG"
    m.close()


def test_launch_count_diagonal_vs_sequential(small):
    cfg, w, _, _ = small
    from recurrent_memory_transformer_diag_b200 import Armt
    m = Armt(cfg)
    S, L = cfg.n_segments, cfg.n_layers
    m.set_schedule("diagonal")
    nd = m.launch_count(S)
    m.set_schedule("sequential")
    ns = m.launch_count(S)
    m.close()
    assert nd < ns
    # every wave launches the same kernel sequence (b kernels), plus extra
    # kernels in the S waves that hold a layer-0 node (and, where the output
    # is not fused, the S waves that hold a last-layer node): the same extras
    # in both schedules, so ns - nd = (S*L - (S+L-1)) * b
    b, rem = divmod(ns - nd, S * L - (S + L - 1))
    assert rem == 0 and b > 0
    extra = nd - (S + L - 1) * b
    assert extra in (S, 2 * S)
    assert ns == S * L * b + extra
