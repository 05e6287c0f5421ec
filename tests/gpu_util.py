"""Helpers of the GPU tests: run the library forward on torch device buffers."""
import numpy as np


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def run_gpu(cfg, weights, emb, S, schedule="diagonal", graph=True, max_segments=None, repeat=1,
            model=None):
    """Forward through the C ABI; returns (hidden fp32, A, z) as numpy arrays."""
    import torch
    from recurrent_memory_transformer_diag_b200 import Armt
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    T, L, d, P = cfg.seg_len, cfg.n_layers, cfg.d_model, cfg.phi_dim
    m = model or Armt(cfg, max_segments=max_segments or S, schedule=schedule)
    if model is None:
        m.load_weights(weights)
    m.set_schedule(schedule)
    m.set_graph(graph)
    e = torch.from_numpy(np.ascontiguousarray(emb)).to("cuda").to(dt)
    out = torch.empty(S * T, d, dtype=dt, device="cuda")
    A = torch.empty(L, d, P, dtype=torch.float32, device="cuda")
    z = torch.empty(L, P, dtype=torch.float32, device="cuda")
    for _ in range(repeat):
        m.forward(e, S, T, out, A, z)
    m.device_status()
    torch.cuda.synchronize()
    res = (out.float().cpu().numpy(), A.cpu().numpy(), z.cpu().numpy())
    if model is None:
        m.close()
    return res
