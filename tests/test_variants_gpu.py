"""ARMT write variants and streaming resume on the GPU, against the oracle.

* Gated write (row j's change of A scaled by sigmoid(w_beta . m_j)) and
  unclamped gamma, each alone and together: tiny (fp32, rel-L2 <= 1e-5) and
  small (bf16 mode, <= 1e-2), per segment and per layer.
* armt_forward_ex with carry_state: S1 segments, then the next S2 from the
  carried (A, z), equal S1 + S2 segments in one call bit for bit (every node
  runs the same kernels on the same inputs in both), and match the oracle
  started from the same state.
"""
import numpy as np
import pytest

import oracle
from recurrent_memory_transformer_diag_b200.inputs import CONFIGS, make_embeddings, make_weights

from .gpu_util import rel_l2, run_gpu
from .test_parity_scale_gpu import per_part_errors

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-5, "bf16": 1e-2}


@pytest.mark.parametrize("name", ["tiny", "small"])
@pytest.mark.parametrize("gate,clamp", [(True, True), (False, False), (True, False)])
def test_write_variants_match_oracle(name, gate, clamp):
    cfg = CONFIGS[name].with_(write_gate=gate, gamma_clamp=clamp)
    S = cfg.n_segments
    w = make_weights(cfg)
    emb = make_embeddings(cfg, S)
    ref = oracle.forward(cfg, w, emb)
    got = run_gpu(cfg, w, emb, S)
    errs = per_part_errors(cfg, got, ref, S)
    worst = max(errs, key=errs.get)
    print(f"\n{name} gate={gate} clamp={clamp}: worst {worst} {errs[worst]:.3e}")
    bad = {k: v for k, v in errs.items() if not v <= TOL[cfg.dtype]}
    assert not bad, bad
    plain = oracle.forward(CONFIGS[name], w, emb)
    assert rel_l2(ref[1], plain[1]) > 10 * TOL[cfg.dtype]    # the variant is visible in the state


@pytest.mark.parametrize("name,split", [("tiny", 1), ("small", 5)])
@pytest.mark.parametrize("schedule", ["diagonal", "sequential"])
def test_streaming_resume_equals_one_call(name, split, schedule):
    import torch
    from recurrent_memory_transformer_diag_b200 import Armt
    cfg = CONFIGS[name]
    S, T, L, d, P = cfg.n_segments, cfg.seg_len, cfg.n_layers, cfg.d_model, cfg.phi_dim
    w = make_weights(cfg)
    emb_h = make_embeddings(cfg, S)
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    emb = torch.from_numpy(emb_h).cuda().to(dt)
    m = Armt(cfg, max_segments=S, schedule=schedule)
    m.load_weights(w)
    out = torch.empty(S * T, d, dtype=dt, device="cuda")
    A = torch.empty(L, d, P, device="cuda")
    z = torch.empty(L, P, device="cuda")
    m.forward(emb, S, T, out, A, z)
    # two calls: segments [0, split) from zero state, then [split, S) carried
    out2 = torch.empty_like(out)
    A2 = torch.full_like(A, float("nan"))
    z2 = torch.full_like(z, float("nan"))
    m.forward_ex(emb, split, T, out2, A2, z2, carry_state=False)
    m.forward_ex(emb[split * T:], S - split, T, out2[split * T:], A2, z2, carry_state=True)
    m.device_status()
    torch.cuda.synchronize()
    for x, y in ((out, out2), (A, A2), (z, z2)):
        np.testing.assert_array_equal(x.float().cpu().numpy(), y.float().cpu().numpy())
    # the second call alone against the oracle started from the first call's state
    A1 = torch.empty_like(A)
    z1 = torch.empty_like(z)
    out1 = torch.empty_like(out)
    m.forward(emb, split, T, out1, A1, z1)
    torch.cuda.synchronize()
    A1h, z1h = A1.cpu().numpy().astype(np.float64), z1.cpu().numpy().astype(np.float64)
    ref = oracle.forward(cfg, w, emb_h[split * T:], A0=A1h, z0=z1h)
    got = (out2[split * T:].float().cpu().numpy(), A2.cpu().numpy(), z2.cpu().numpy())
    errs = per_part_errors(cfg, got, ref, S - split)
    worst = max(errs, key=errs.get)
    print(f"\n{name} resume at {split} ({schedule}): worst {worst} {errs[worst]:.3e}")
    bad = {k: v for k, v in errs.items() if not v <= TOL[cfg.dtype]}
    assert not bad, bad
    m.close()


def test_forward_ex_rejects_bad_flag():
    import torch
    from recurrent_memory_transformer_diag_b200 import Armt, ArmtError
    cfg = CONFIGS["tiny"]
    m = Armt(cfg)
    m.load_weights(make_weights(cfg))
    e = torch.zeros(cfg.seg_len, cfg.d_model, device="cuda")
    A = torch.zeros(cfg.n_layers, cfg.d_model, cfg.phi_dim, device="cuda")
    z = torch.zeros(cfg.n_layers, cfg.phi_dim, device="cuda")
    from recurrent_memory_transformer_diag_b200.armt import lib, _ptr
    st = torch.cuda.current_stream().cuda_stream
    assert lib().armt_forward_ex(m._h, _ptr(e), 1, cfg.seg_len, _ptr(e), _ptr(A), _ptr(z), 2, st) == 1
    m.close()
    del ArmtError
