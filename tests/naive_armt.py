"""Brute-force restatement of the ARMT recurrence in pure-Python loops.

Used only to pin the oracle on tiny inputs.  It is written independently of
``oracle/`` (no numpy arithmetic, nothing imported from it) and formulates
each step differently: RoPE as complex multiplication, attention as explicit
per-query loops, DPFP with explicit index arithmetic, the delta rule one
scalar at a time.  The readings it follows are the same ones the oracle
states (pre-norm LLaMA layer; ARMT read before and delta-rule write after the
layer, the write taking the RMS-normalised memory rows one after another;
memory tokens appended to every segment).
"""
import cmath
import math


def _mat(a):
    return [list(map(float, r)) for r in a]


def _linear(x, w):
    """x [T][in], w [out][in] (nn.Linear layout) -> [T][out]."""
    return [[sum(xr[i] * wr[i] for i in range(len(xr))) for wr in w] for xr in x]


def _rmsnorm(x, g, eps):
    out = []
    for r in x:
        ms = sum(v * v for v in r) / len(r)
        inv = 1.0 / math.sqrt(ms + eps)
        out.append([r[i] * inv * g[i] for i in range(len(r))])
    return out


def _rope_row(vec, pos, theta):
    hd = len(vec)
    half = hd // 2
    out = list(vec)
    for j in range(half):
        c = complex(vec[j], vec[j + half]) * cmath.exp(1j * pos * theta ** (-2.0 * j / hd))
        out[j], out[j + half] = c.real, c.imag
    return out


def _dpfp(x, nu):
    n2 = 2 * len(x)
    r = [max(v, 0.0) for v in x] + [max(-v, 0.0) for v in x]
    phi = []
    for n in range(1, nu + 1):
        for j in range(n2):
            phi.append(r[j] * r[(j - n) % n2])
    return phi


def _layer(x, W, l, cfg):
    T = len(x)
    H, KV, hd = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    xn = _rmsnorm(x, W["attn_norm"][l], cfg.rms_eps)
    q = _linear(xn, W["wq"][l])
    k = _linear(xn, W["wk"][l])
    v = _linear(xn, W["wv"][l])
    for t in range(T):
        for h in range(H):
            q[t][h * hd:(h + 1) * hd] = _rope_row(q[t][h * hd:(h + 1) * hd], t, cfg.rope_theta)
        for h in range(KV):
            k[t][h * hd:(h + 1) * hd] = _rope_row(k[t][h * hd:(h + 1) * hd], t, cfg.rope_theta)
    o = [[0.0] * (H * hd) for _ in range(T)]
    group = H // KV
    for h in range(H):
        g = h // group
        for t in range(T):
            sc = []
            for u in range(t + 1):
                dot = sum(q[t][h * hd + e] * k[u][g * hd + e] for e in range(hd))
                sc.append(dot / math.sqrt(hd))
            mx = max(sc)
            ex = [math.exp(s - mx) for s in sc]
            tot = sum(ex)
            for e in range(hd):
                o[t][h * hd + e] = sum(ex[u] * v[u][g * hd + e] for u in range(t + 1)) / tot
    ao = _linear(o, W["wo"][l])
    x = [[x[t][i] + ao[t][i] for i in range(len(x[t]))] for t in range(T)]
    xn = _rmsnorm(x, W["mlp_norm"][l], cfg.rms_eps)
    gt = _linear(xn, W["w_gate"][l])
    up = _linear(xn, W["w_up"][l])
    u = [[(gt[t][f] / (1.0 + math.exp(-gt[t][f]))) * up[t][f] for f in range(len(gt[t]))]
         for t in range(T)]
    dn = _linear(u, W["w_down"][l])
    return [[x[t][i] + dn[t][i] for i in range(len(x[t]))] for t in range(T)]


def forward(cfg, weights, emb, memory=True, A0=None, z0=None):
    """Segment-major recurrence; returns (hidden [S*T][d], A [L][d][P], z [L][P]).
    The write variants follow cfg.write_gate (row j's change of A times
    1 / (1 + exp(-w_beta . m_j))) and cfg.gamma_clamp; (A0, z0) is the state
    to start from (zeros when not given)."""
    W = {}
    for name, arr in weights.items():
        if arr.ndim == 1:
            W[name] = list(map(float, arr))
        elif arr.ndim == 2:
            W[name] = _mat(arr)
        else:
            W[name] = [_mat(a) for a in arr]
    T, L, d, M = cfg.seg_len, cfg.n_layers, cfg.d_model, cfg.n_mem
    P = 2 * cfg.d_key * cfg.dpfp_nu
    eps = cfg.mem_eps
    S = len(emb) // T
    A = [[[0.0] * P for _ in range(d)] for _ in range(L)]
    z = [[0.0] * P for _ in range(L)]
    if A0 is not None:
        A = [[[float(A0[l][i][p]) for p in range(P)] for i in range(d)] for l in range(L)]
        z = [[float(z0[l][p]) for p in range(P)] for l in range(L)]
    gate = getattr(cfg, "write_gate", False)
    clamp = getattr(cfg, "gamma_clamp", True)
    hidden = []
    for s in range(S):
        x = _mat(emb[s * T:(s + 1) * T]) + [list(r) for r in W["mem_emb"]]
        for l in range(L):
            if memory:
                q = _linear(x, W["wq_mem"][l])
                for t in range(len(x)):
                    phi = _dpfp(q[t], cfg.dpfp_nu)
                    den = sum(z[l][p] * phi[p] for p in range(P)) + eps
                    for i in range(d):
                        x[t][i] += sum(A[l][i][p] * phi[p] for p in range(P)) / den
            x = _layer(x, W, l, cfg)
            if memory:
                mem = _rmsnorm(x[T:T + M], [1.0] * d, cfg.rms_eps)
                kk = _linear(mem, W["wk_mem"][l])
                vv = _linear(mem, W["wv_mem"][l])
                for j in range(M):              # one memory row after another
                    phi = _dpfp(kk[j], cfg.dpfp_nu)
                    zphi = sum(z[l][p] * phi[p] for p in range(P))
                    nrm = sum(p * p for p in phi)
                    gamma = 1.0 - zphi / (nrm + eps)
                    if clamp:
                        gamma = min(max(gamma, 0.0), 1.0)
                    beta = 1.0
                    if gate:
                        beta = 1.0 / (1.0 + math.exp(-sum(W["w_beta"][l][i] * mem[j][i] for i in range(d))))
                    for i in range(d):
                        vbar = sum(A[l][i][p] * phi[p] for p in range(P)) / (zphi + eps)
                        for p in range(P):
                            A[l][i][p] += beta * (vv[j][i] - vbar) * phi[p]
                    for p in range(P):
                        z[l][p] += gamma * phi[p]
        hidden.extend(x[:T])
    return hidden, A, z
