"""Model shapes and seeded synthetic inputs for the ARMT forward.

This module holds no part of the method's arithmetic: it only names the
shapes of the workloads and draws random tensors for them.  Both the CUDA
path (through the C-ABI) and the CPU oracle are fed from here, so that they
see bit-identical inputs.

Workloads (Diagonal Batching paper, Fig. 1 and abstract: LLaMA-1B ARMT,
131072 tokens, segment 1024; ARMT is the layer-recurrent model the method
targets):

* ``tiny``  fp32:  L=2,  d=64,   4x16 heads,        ffn 172,  M=4,  T=16,   S=4
* ``small`` bf16:  L=4,  d=256,  4x64 heads,        ffn 688,  M=16, T=128,  S=16
* ``1b``    bf16:  L=16, d=2048, 32x64 / 8 KV,      ffn 8192, M=16, T=1024, S=128
* ``3b``    bf16:  L=28, d=3072, 24x128 / 8 KV,     ffn 8192, M=16, T=2048, S=32

Value distributions: linear weights and memory-token embeddings N(0, 0.02),
input embeddings N(0, 1), RMSNorm gains 1 (optionally 1 + 0.1 N(0, 1) in
tests).  In bf16 workloads every tensor is
rounded (round-to-nearest-even) to a bf16-representable fp32 value here, so
that the oracle computes on exactly the values the GPU loads.

Random numbers come from PyTorch's CPU generator (``torch.Generator`` seeded
per tensor), a fixed, published algorithm, so the draws are reproducible on
every host with the same PyTorch release.
"""
from __future__ import annotations

import dataclasses
from typing import Dict

import numpy as np

WEIGHT_SEED = 1234
EMB_SEED = 5678

# Order fixes each tensor's seed offset; never reorder (new tensors go last).
WEIGHT_NAMES = (
    "mem_emb", "attn_norm", "mlp_norm", "wq", "wk", "wv", "wo",
    "w_gate", "w_up", "w_down", "wq_mem", "wk_mem", "wv_mem", "w_beta",
)


@dataclasses.dataclass(frozen=True)
class ArmtConfig:
    name: str
    n_layers: int
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    d_ffn: int
    n_mem: int
    d_key: int
    dpfp_nu: int
    seg_len: int
    n_segments: int
    dtype: str = "bf16"          # "fp32" or "bf16": weights/activations; state is fp32
    rope_theta: float = 500000.0
    rms_eps: float = 1e-5
    mem_eps: float = 1e-5
    write_gate: bool = False     # ARMT variant: row j's write of A scaled by sigmoid(w_beta . m_j)
    gamma_clamp: bool = True     # ARMT variant: False leaves gamma_j unclamped

    @property
    def phi_dim(self) -> int:
        """P = 2 * d_key * nu, the DPFP feature dimension."""
        return 2 * self.d_key * self.dpfp_nu

    @property
    def rows(self) -> int:
        """T' = T + M rows processed per (segment, layer) node."""
        return self.seg_len + self.n_mem

    @property
    def n_tokens(self) -> int:
        return self.seg_len * self.n_segments

    def with_(self, **kw) -> "ArmtConfig":
        return dataclasses.replace(self, **kw)

    def weight_shapes(self) -> Dict[str, tuple]:
        L, d, H, KV, hd, F = (self.n_layers, self.d_model, self.n_heads,
                              self.n_kv_heads, self.head_dim, self.d_ffn)
        dk = self.d_key
        return {
            "mem_emb": (self.n_mem, d),
            "attn_norm": (L, d),
            "mlp_norm": (L, d),
            "wq": (L, H * hd, d),
            "wk": (L, KV * hd, d),
            "wv": (L, KV * hd, d),
            "wo": (L, d, H * hd),
            "w_gate": (L, F, d),
            "w_up": (L, F, d),
            "w_down": (L, d, F),
            "wq_mem": (L, dk, d),
            "wk_mem": (L, dk, d),
            "wv_mem": (L, d, d),
            **({"w_beta": (L, d)} if self.write_gate else {}),
        }


CONFIGS: Dict[str, ArmtConfig] = {
    "tiny": ArmtConfig("tiny", n_layers=2, d_model=64, n_heads=4, n_kv_heads=4, head_dim=16,
                       d_ffn=172, n_mem=4, d_key=16, dpfp_nu=2, seg_len=16, n_segments=4,
                       dtype="fp32"),
    "small": ArmtConfig("small", n_layers=4, d_model=256, n_heads=4, n_kv_heads=4, head_dim=64,
                        d_ffn=688, n_mem=16, d_key=64, dpfp_nu=3, seg_len=128, n_segments=16),
    "1b": ArmtConfig("1b", n_layers=16, d_model=2048, n_heads=32, n_kv_heads=8, head_dim=64,
                     d_ffn=8192, n_mem=16, d_key=64, dpfp_nu=3, seg_len=1024, n_segments=128),
    "3b": ArmtConfig("3b", n_layers=28, d_model=3072, n_heads=24, n_kv_heads=8, head_dim=128,
                     d_ffn=8192, n_mem=16, d_key=128, dpfp_nu=3, seg_len=2048, n_segments=32),
}


def _randn(shape, seed: int, std: float) -> np.ndarray:
    import torch
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    t = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t


def _round(t, dtype: str) -> np.ndarray:
    import torch
    if dtype == "bf16":
        t = t.to(torch.bfloat16).to(torch.float32)
    return np.ascontiguousarray(t.numpy())


def make_weights(cfg: ArmtConfig, seed: int = WEIGHT_SEED, std: float = 0.02,
                 gain_std: float = 0.0) -> Dict[str, np.ndarray]:
    """All weights of ``cfg`` as host fp32 arrays, nn.Linear layout [out, in].

    RMSNorm gains are 1 by default; ``gain_std > 0`` draws them as
    1 + gain_std * N(0, 1) instead (a test input that makes a slip in how the
    gains reach the projections visible)."""
    import torch
    out = {}
    shapes = cfg.weight_shapes()
    for k, name in enumerate(WEIGHT_NAMES):
        if name not in shapes:
            continue
        shape = shapes[name]
        if name in ("attn_norm", "mlp_norm"):
            t = torch.ones(*shape, dtype=torch.float32)
            if gain_std > 0:
                t = t + _randn(shape, seed * 1000 + k, gain_std)
        else:
            t = _randn(shape, seed * 1000 + k, std)
        out[name] = _round(t, cfg.dtype)
    return out


def make_embeddings(cfg: ArmtConfig, n_segments: int | None = None, seed: int = EMB_SEED) -> np.ndarray:
    """Input embeddings [S*T, d], N(0, 1).  A prefix of S' segments equals the
    first S'*T rows of the full draw (the draw is made for cfg.n_segments)."""
    S = cfg.n_segments if n_segments is None else n_segments
    full = max(S, cfg.n_segments)
    t = _randn((full * cfg.seg_len, cfg.d_model), seed, 1.0)
    return _round(t[: S * cfg.seg_len].contiguous(), cfg.dtype)
