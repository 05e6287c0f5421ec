"""Oracle: plain fp64 CPU forward of a layer-recurrent ARMT over S segments.

TEST INFRASTRUCTURE ONLY.  It is slow on purpose and shares no code with the
CUDA path: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import it.  Numpy matrix products serve as library
steps; there is no blocking, fusion or reordering beyond the definitions
below.

What the pages fix
------------------
* The recurrence and its order.  Node (s, l) reads only the output of
  (s, l-1) and the per-layer memory state left by (s-1, l); running the nodes
  segment-major (S x L steps) or by diagonals s + l = i computes the same
  thing ("Diagonal Batching for Recurrent Memory Transformers" skill page,
  "Practical Guidance"; Pith review of arXiv 2506.05229, "What carries the
  argument" and "Core claim": each layer keeps its own memory and updates it
  once per segment).
* The model family: an ARMT (associative recurrent memory transformer) built
  on a LLaMA-1B-shaped decoder (Pith review, "The reading"; Figure 1 caption).
* Memory tokens concatenated to every segment (Figure 2 caption).

What the pages leave open, and the reading taken here
-----------------------------------------------------
The pages give no layer equations.  The readings below are the plainest ones
consistent with the model family the pages name (LLaMA decoder; ARMT with a
DPFP feature map [Schlag et al., ref. 29] and a delta-rule write [ref. 38],
both cited in the Pith review's reference list):

1. Segment input (layer 0): the T embeddings of segment s followed by the M
   memory-token embeddings (the same M rows every segment).  T' = T + M rows
   flow through all layers.
2. Memory read, before the layer: q = X Wq_mem^T; phi = DPFP_nu(q);
   X <- X + (phi A^T) / (phi . z + eps), for all T' rows, with the state
   (A_l, z_l) left by segment s-1 (zero for segment 0, so the read adds 0).
3. Pre-norm LLaMA layer: X <- X + Attn(RMSNorm(X) g_attn); X <- X + MLP(RMSNorm(X) g_mlp)
   with rotate-half RoPE (pairs j, j+hd/2; inv_freq_j = theta^(-2j/hd);
   positions 0..T'-1, restarting every segment), causal softmax attention
   over the T' rows of this node only, scale 1/sqrt(hd), query head h using
   kv head floor(h * KV / H), and MLP = (silu(x Wg^T) * (x Wu^T)) Wd^T.
4. Memory write, after the layer, from the M memory rows of the layer
   output (rows T..T'-1), each RMS-normalised without gain (m = RMSNorm(row)):
   k = m Wk_mem^T, v = m Wv_mem^T, phi_j = DPFP(k_j), and the delta rule
   applied to the rows one after another (j = 0..M-1), each seeing the state
   the previous rows left:
     vbar_j  = A phi_j / (z . phi_j + eps)
     gamma_j = clamp(1 - (z . phi_j) / (|phi_j|^2 + eps), 0, 1)
     A <- A + (v_j - vbar_j) phi_j^T;   z <- z + gamma_j phi_j
   The memory is updated once per segment (after the segment's layer), the
   M rows in order: the delta rule is a sequential recurrence (ref. 38
   parallelises exactly that recurrence).  Applying all M rows to the
   pre-write state at once, or writing un-normalised rows, makes this
   random-init model diverge geometrically over the segments (fp64: hidden
   RMS x2 and |A| x10 per segment at the 1B shape), so no finite-precision
   forward over 128 segments could be compared with it.
   Two variants of the write, both off by default (the ARMT family the
   Pith review names, ref. 28, and the delta rule, ref. 38, have them; the
   pages print neither):
     gated write:      A <- A + beta_j (v_j - vbar_j) phi_j^T with
                       beta_j = sigmoid(w_beta[l] . m_j), z as above;
     unclamped gamma:  gamma_j = 1 - (z . phi_j) / (|phi_j|^2 + eps).
   And the state a forward starts from may be given (A0, z0) instead of 0:
   a long input streamed over several calls carries the state across them.
5. DPFP_nu(x): r = [relu(x); relu(-x)] (length 2 d_k);
   phi[(n-1) 2 d_k + j] = r_j * r_{(j-n) mod 2 d_k}, n = 1..nu  (P = 2 d_k nu).
6. Output: rows 0..T-1 of node (s, L-1) are the final hidden states of
   segment s; after all segments, A_l and z_l of every layer.
"""
from __future__ import annotations

from typing import Dict, Iterable, Optional, Sequence, Tuple

import numpy as np

from .schedule import diagonal_waves

F64 = np.float64


# ---------------------------------------------------------------------------
# building blocks (readings 2-5)
# ---------------------------------------------------------------------------

def rms_norm(x: np.ndarray, gain: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * gain, per row."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * gain


def rope_cos_sin(n_pos: int, head_dim: int, theta: float) -> Tuple[np.ndarray, np.ndarray]:
    """cos/sin of angle p * theta^(-2j/hd), p < n_pos, j < hd/2."""
    j = np.arange(head_dim // 2, dtype=F64)
    inv_freq = theta ** (-2.0 * j / head_dim)
    ang = np.arange(n_pos, dtype=F64)[:, None] * inv_freq[None, :]
    return np.cos(ang), np.sin(ang)


def apply_rope(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Rotate pairs (j, j + hd/2) of x [T', heads, hd] by the angles of their row."""
    half = x.shape[-1] // 2
    x1, x2 = x[..., :half], x[..., half:]
    c, s = cos[:, None, :], sin[:, None, :]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def causal_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """q [T', H, hd], k/v [T', KV, hd] -> [T', H, hd]; row t attends to rows <= t."""
    T, H, hd = q.shape
    KV = k.shape[1]
    out = np.empty_like(q)
    mask = np.triu(np.ones((T, T), dtype=bool), k=1)
    for h in range(H):
        g = (h * KV) // H
        sc = (q[:, h, :] @ k[:, g, :].T) / np.sqrt(hd)
        sc[mask] = -np.inf
        sc = sc - sc.max(axis=-1, keepdims=True)
        p = np.exp(sc)
        p /= p.sum(axis=-1, keepdims=True)
        out[:, h, :] = p @ v[:, g, :]
    return out


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def dpfp(x: np.ndarray, nu: int) -> np.ndarray:
    """Deterministic parameter-free projection of order nu along the last axis."""
    r = np.concatenate([np.maximum(x, 0.0), np.maximum(-x, 0.0)], axis=-1)
    return np.concatenate([r * np.roll(r, n, axis=-1) for n in range(1, nu + 1)], axis=-1)


def mem_read(x: np.ndarray, wq_mem: np.ndarray, A: np.ndarray, z: np.ndarray,
             nu: int, eps: float) -> np.ndarray:
    """Retrieved value r for every row of x [T', d]; A [d, P], z [P]."""
    phi = dpfp(x @ wq_mem.T, nu)                  # [T', P]
    return (phi @ A.T) / (phi @ z + eps)[:, None]


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def mem_write(m: np.ndarray, wk_mem: np.ndarray, wv_mem: np.ndarray, A: np.ndarray,
              z: np.ndarray, nu: int, eps: float, w_beta: Optional[np.ndarray] = None,
              clamp_gamma: bool = True) -> Tuple[np.ndarray, np.ndarray]:
    """Delta-rule update of (A, z) from memory rows m [M, d], row after row;
    returns the new (A, z).  ``w_beta`` [d] gates each row's write of A by
    sigmoid(w_beta . m_j); ``clamp_gamma=False`` leaves gamma unclamped."""
    k = m @ wk_mem.T                              # [M, dk]
    v = m @ wv_mem.T                              # [M, d]
    phi = dpfp(k, nu)                             # [M, P]
    beta = sigmoid(m @ w_beta) if w_beta is not None else np.ones(m.shape[0])
    A = A.copy()
    z = z.copy()
    for j in range(m.shape[0]):
        zphi = phi[j] @ z
        vbar = (A @ phi[j]) / (zphi + eps)
        gamma = 1.0 - zphi / (phi[j] @ phi[j] + eps)
        if clamp_gamma:
            gamma = min(max(gamma, 0.0), 1.0)
        A += beta[j] * np.outer(v[j] - vbar, phi[j])
        z += gamma * phi[j]
    return A, z


def decoder_layer(x: np.ndarray, w: Dict[str, np.ndarray], l: int, cfg) -> np.ndarray:
    """One pre-norm LLaMA layer on the T' rows of one node (reading 3)."""
    T = x.shape[0]
    H, KV, hd = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    xn = rms_norm(x, w["attn_norm"][l], cfg.rms_eps)
    q = (xn @ w["wq"][l].T).reshape(T, H, hd)
    k = (xn @ w["wk"][l].T).reshape(T, KV, hd)
    v = (xn @ w["wv"][l].T).reshape(T, KV, hd)
    cos, sin = rope_cos_sin(T, hd, cfg.rope_theta)
    q, k = apply_rope(q, cos, sin), apply_rope(k, cos, sin)
    o = causal_attention(q, k, v).reshape(T, H * hd)
    x = x + o @ w["wo"][l].T
    xn = rms_norm(x, w["mlp_norm"][l], cfg.rms_eps)
    u = silu(xn @ w["w_gate"][l].T) * (xn @ w["w_up"][l].T)
    return x + u @ w["w_down"][l].T


def node_forward(x: np.ndarray, w: Dict[str, np.ndarray], l: int, A: np.ndarray,
                 z: np.ndarray, cfg, memory: bool = True):
    """Node (s, l): read (with the state of segment s-1), layer, write.
    Returns (layer output [T', d], new A_l, new z_l).  ``memory=False`` skips
    the read and the write (a test hook: each segment then is an independent
    LLaMA forward)."""
    if memory:
        x = x + mem_read(x, w["wq_mem"][l], A, z, cfg.dpfp_nu, cfg.mem_eps)
    x = decoder_layer(x, w, l, cfg)
    if memory:
        m = rms_norm(x[cfg.seg_len:], np.ones(x.shape[1]), cfg.rms_eps)
        w_beta = w["w_beta"][l] if getattr(cfg, "write_gate", False) else None
        A, z = mem_write(m, w["wk_mem"][l], w["wv_mem"][l], A, z, cfg.dpfp_nu, cfg.mem_eps,
                         w_beta=w_beta, clamp_gamma=getattr(cfg, "gamma_clamp", True))
    return x, A, z


# ---------------------------------------------------------------------------
# the recurrence (readings 1 and 6)
# ---------------------------------------------------------------------------

def forward(cfg, weights: Dict[str, np.ndarray], emb: np.ndarray,
            order: Optional[Iterable[Tuple[int, int]]] = None, memory: bool = True,
            A0: Optional[np.ndarray] = None, z0: Optional[np.ndarray] = None):
    """Run every node of S = len(emb) / T segments in ``order`` (default:
    segment-major).  Each node must come after its two predecessors.  The
    memory state starts from (A0, z0) when given (the state a previous call
    left), else from 0.

    Returns (hidden [S*T, d], A [L, d, P], z [L, P]) in fp64.
    """
    T, L, d, P = cfg.seg_len, cfg.n_layers, cfg.d_model, cfg.phi_dim
    emb = np.asarray(emb, dtype=F64)
    assert emb.shape[0] % T == 0 and emb.shape[1] == d
    S = emb.shape[0] // T
    w = {k: np.asarray(v, dtype=F64) for k, v in weights.items()}
    if order is None:
        order = [(s, l) for s in range(S) for l in range(L)]
    A = np.zeros((L, d, P), dtype=F64) if A0 is None else np.array(A0, dtype=F64)
    z = np.zeros((L, P), dtype=F64) if z0 is None else np.array(z0, dtype=F64)
    assert A.shape == (L, d, P) and z.shape == (L, P)
    hidden = np.zeros((S * T, d), dtype=F64)
    cur: Dict[int, np.ndarray] = {}     # output of the latest layer run, per segment
    done_layer = np.full(S, -1)         # latest layer run, per segment
    done_seg = np.full(L, -1)           # latest segment whose write reached A_l
    for s, l in order:
        if done_layer[s] != l - 1 or done_seg[l] != s - 1:
            raise ValueError(f"node {(s, l)} scheduled before a predecessor")
        if l == 0:
            x = np.concatenate([emb[s * T:(s + 1) * T], w["mem_emb"]], axis=0)
        else:
            x = cur[s]
        x, A[l], z[l] = node_forward(x, w, l, A[l], z[l], cfg, memory=memory)
        cur[s] = x
        done_layer[s] = l
        done_seg[l] = s
        if l == L - 1:
            hidden[s * T:(s + 1) * T] = x[:T]
            del cur[s]
    if (done_layer != L - 1).any():
        raise ValueError("order left nodes unscheduled")
    return hidden, A, z


def diagonal_order(S: int, L: int) -> Sequence[Tuple[int, int]]:
    """Nodes wave by wave (s + l = i), layers ascending inside a wave."""
    return [n for wave in diagonal_waves(S, L) for n in wave]
