"""armt_stage_wave (the layer-pipelined forward's per-stage call) on one GPU.

Two or three stage contexts, each created with its layer block and loaded
with those layers' weights, run every global wave one after another in this
process; a device copy stands in for the point-to-point hand-off between
ranks (stage g's rows of wave i are stage g + 1's input of wave i + 1).  No
stage waits on another: the waves are enqueued in order on one stream.  The
final hidden states and every layer's A_l, z_l must equal the whole-model
armt_forward bit for bit: each node runs the same kernels on the same inputs.
"""
import numpy as np
import pytest

from recurrent_memory_transformer_diag_b200.inputs import CONFIGS, make_embeddings, make_weights

from .gpu_util import run_gpu

pytestmark = pytest.mark.gpu


def _stage_weights(w, off, cnt):
    return {k: (v if k == "mem_emb" else v[off:off + cnt]) for k, v in w.items()}


def _run_pipeline(cfg, w, emb, S, stages):
    import torch
    from recurrent_memory_transformer_diag_b200 import Armt
    from recurrent_memory_transformer_diag_b200.pipeline import layer_blocks, wave_io
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    T, L, d, P, Tp = cfg.seg_len, cfg.n_layers, cfg.d_model, cfg.phi_dim, cfg.seg_len + cfg.n_mem
    blocks = layer_blocks(L, stages)
    models, states = [], []
    for off, cnt in blocks:
        m = Armt(cfg.with_(n_layers=cnt), max_segments=S)
        m.load_weights(_stage_weights(w, off, cnt))
        models.append(m)
        states.append((torch.empty(cnt, d, P, dtype=torch.float32, device="cuda"),
                       torch.empty(cnt, P, dtype=torch.float32, device="cuda")))
    e = torch.from_numpy(np.ascontiguousarray(emb)).to("cuda").to(dt)
    out = torch.full((S * T, d), float("nan"), dtype=dt, device="cuda")
    inbox = [torch.zeros(Tp, d, dtype=torch.float32, device="cuda") for _ in blocks]
    outbox = [torch.zeros(Tp, d, dtype=torch.float32, device="cuda") for _ in blocks]
    for i in range(S + L - 1):
        sent = []
        for g, ((off, cnt), m) in enumerate(zip(blocks, models)):
            recv, send = wave_io(i, S, off, cnt, L)
            A, z = states[g]
            m.stage_wave(S, T, i, off, L, e, inbox[g] if recv else None, outbox[g] if send else None,
                         out, A, z)
            if send:
                sent.append(g)
        for g in sent:   # the hand-off: received by the next stage in the next wave
            inbox[g + 1].copy_(outbox[g])
    for m in models:
        m.device_status()
    torch.cuda.synchronize()
    A = np.concatenate([a.cpu().numpy() for a, _ in states])
    z = np.concatenate([zz.cpu().numpy() for _, zz in states])
    for m in models:
        m.close()
    return out.float().cpu().numpy(), A, z


@pytest.mark.parametrize("name,S,stages", [("small", 5, 2), ("small", 6, 3), ("tiny", 4, 2)])
def test_stage_waves_equal_the_whole_forward(name, S, stages):
    cfg = CONFIGS[name]
    w = make_weights(cfg)
    emb = make_embeddings(cfg, S)
    ref = run_gpu(cfg, w, emb, S)
    got = _run_pipeline(cfg, w, emb, S, stages)
    for x, y in zip(got, ref):
        np.testing.assert_array_equal(x, y)


def test_stage_wave_rejects_missing_handoff_buffers():
    import torch
    from recurrent_memory_transformer_diag_b200 import Armt, ArmtError
    cfg = CONFIGS["small"]
    w = make_weights(cfg)
    m = Armt(cfg.with_(n_layers=2), max_segments=4)
    m.load_weights(_stage_weights(w, 2, 2))
    d, P, T = cfg.d_model, cfg.phi_dim, cfg.seg_len
    A = torch.empty(2, d, P, device="cuda")
    z = torch.empty(2, P, device="cuda")
    out = torch.empty(4 * T, d, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ArmtError):   # wave 2 holds node (0, 2): its input rows are needed
        m.stage_wave(4, T, 2, 2, 4, None, None, None, out, A, z)
    with pytest.raises(ArmtError):   # a block past the model's last layer
        m.stage_wave(4, T, 0, 3, 4, None, None, None, out, A, z)
    with pytest.raises(ArmtError):   # a wave past the last one
        m.stage_wave(4, T, 7, 2, 4, None, None, None, out, A, z)
    m.close()
