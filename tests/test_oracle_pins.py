"""Pins of the fp64 oracle against values fixed outside it.

Each test checks one oracle function against a hand-computed value
(tests/golden), a closed form, an invariant, or the pure-Python brute force
in tests/naive_armt.py.  The mutation tests at the end plant plausible
mistakes in the oracle (on the CPU) and check that some pin catches each.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import armt_oracle as ao
from recurrent_memory_transformer_diag_b200.inputs import CONFIGS, ArmtConfig, make_embeddings, make_weights

from . import naive_armt

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(7)


def _micro(**kw):
    base = dict(name="micro", n_layers=2, d_model=8, n_heads=2, n_kv_heads=1, head_dim=4,
                d_ffn=6, n_mem=2, d_key=2, dpfp_nu=2, seg_len=3, n_segments=3, dtype="fp32")
    base.update(kw)
    return ArmtConfig(**base)


def _micro_weights(cfg, seed=3, std=0.3):
    rng = np.random.default_rng(seed)
    w = {}
    for name, shape in cfg.weight_shapes().items():
        if name in ("attn_norm", "mlp_norm"):
            w[name] = 1.0 + 0.2 * rng.standard_normal(shape)
        else:
            w[name] = std * rng.standard_normal(shape)
    return w


# --------------------------------------------------------------------------- DPFP

def test_dpfp_hand_values():
    g = json.load(open(os.path.join(GOLDEN, "dpfp_hand.json")))
    for case in g["cases"]:
        phi = oracle.dpfp(np.array(case["x"]), case["nu"])
        np.testing.assert_array_equal(phi, np.array(case["phi"]), err_msg=case["work"])


def test_dpfp_shape_nonneg_and_dk1_is_zero():
    x = RNG.standard_normal((5, 16))
    phi = oracle.dpfp(x, 3)
    assert phi.shape == (5, 2 * 16 * 3) and (phi >= 0).all()
    assert not oracle.dpfp(RNG.standard_normal((7, 1)), 1).any()


def test_dpfp_positive_homogeneous_degree_two():
    x = RNG.standard_normal(9)
    np.testing.assert_allclose(oracle.dpfp(2.5 * x, 2), 6.25 * oracle.dpfp(x, 2), rtol=1e-14)


# --------------------------------------------------------------------------- delta rule

def _identity_memory(dk):
    return np.eye(dk), np.eye(dk)


def test_single_write_into_empty_state():
    """A=0, z=0: vbar=0, gamma=1, so A = v phi^T and z = phi."""
    dk, nu, eps = 3, 2, 1e-5
    k = np.array([[0.7, -0.4, 1.1]])
    wk, wv = _identity_memory(dk)
    P = 2 * dk * nu
    A, z = oracle.mem_write(k, wk, wv, np.zeros((dk, P)), np.zeros(P), nu, eps)
    phi = oracle.dpfp(k[0], nu)
    np.testing.assert_allclose(A, np.outer(k[0], phi), rtol=0, atol=1e-15)
    np.testing.assert_allclose(z, phi, rtol=0, atol=1e-15)


def test_read_after_write_returns_scaled_value():
    dk, nu, eps = 3, 2, 1e-5
    k = np.array([[0.7, -0.4, 1.1]])
    wk, wv = _identity_memory(dk)
    P = 2 * dk * nu
    A, z = oracle.mem_write(k, wk, wv, np.zeros((dk, P)), np.zeros(P), nu, eps)
    phi = oracle.dpfp(k[0], nu)
    n2 = phi @ phi
    r = oracle.mem_read(k, np.eye(dk), A, z, nu, eps)
    np.testing.assert_allclose(r[0], k[0] * n2 / (n2 + eps), rtol=1e-13)


def test_rewrite_same_key_replaces_value():
    """Writing v then v' under the same key: gamma ~ 0 on the second write and
    the read returns ~v'."""
    dk, nu, eps = 3, 2, 1e-5
    k = np.array([[0.7, -0.4, 1.1]])
    P = 2 * dk * nu
    wk = np.eye(dk)
    A, z = oracle.mem_write(k, wk, np.eye(dk), np.zeros((dk, P)), np.zeros(P), nu, eps)
    wv2 = np.diag([-2.0, 0.5, 3.0])                          # v' = wv2 k
    A2, z2 = oracle.mem_write(k, wk, wv2, A, z, nu, eps)
    phi = oracle.dpfp(k[0], nu)
    n2 = phi @ phi
    gamma = 1.0 - n2 / (n2 + eps)
    np.testing.assert_allclose(z2, z + gamma * phi, rtol=1e-13)
    assert gamma < 1e-4
    r = oracle.mem_read(k, np.eye(dk), A2, z2, nu, eps)
    np.testing.assert_allclose(r[0], wv2 @ k[0], rtol=1e-4)


def test_write_rows_apply_one_after_another():
    """The same key twice in one write: the second row sees the first row's
    state (vbar = v |phi|^2/(|phi|^2+eps), gamma = eps/(|phi|^2+eps)), so the
    value is stored once, not twice (closed form below)."""
    dk, nu, eps = 2, 2, 1e-5
    k = np.array([[0.3, -0.9], [0.3, -0.9]])
    P = 2 * dk * nu
    A, z = oracle.mem_write(k, np.eye(dk), np.eye(dk), np.zeros((dk, P)), np.zeros(P), nu, eps)
    phi = oracle.dpfp(k[0], nu)
    n2 = phi @ phi
    c = n2 / (n2 + eps)
    np.testing.assert_allclose(A, (2.0 - c) * np.outer(k[0], phi), rtol=1e-13)
    np.testing.assert_allclose(z, (1.0 + eps / (n2 + eps)) * phi, rtol=1e-13)


def test_one_write_of_two_rows_equals_two_writes():
    """Sequential reading: writing rows [m1, m2] at once equals writing m1,
    then m2 (the same operations in the same order, up to the matrix
    products' summation order)."""
    rng = np.random.default_rng(11)
    d, dk, nu, eps = 6, 3, 2, 1e-5
    P = 2 * dk * nu
    m = rng.standard_normal((2, d))
    wk, wv = rng.standard_normal((dk, d)), rng.standard_normal((d, d))
    A0, z0 = rng.standard_normal((d, P)) * 0.1, np.abs(rng.standard_normal(P))
    A, z = oracle.mem_write(m, wk, wv, A0, z0, nu, eps)
    A1, z1 = oracle.mem_write(m[:1], wk, wv, A0, z0, nu, eps)
    A2, z2 = oracle.mem_write(m[1:], wk, wv, A1, z1, nu, eps)
    np.testing.assert_allclose(A, A2, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(z, z2, rtol=1e-12, atol=1e-14)


def test_gamma_clamped_at_zero():
    """With z = 2 phi(k) already, writing k gives 1 - z.phi/|phi|^2 ~ -1:
    gamma is clamped to 0 and z stays as it was."""
    dk, nu, eps = 2, 2, 1e-5
    k = np.array([[0.3, -0.9]])
    P = 2 * dk * nu
    z0 = 2 * oracle.dpfp(k[0], nu)
    _, z = oracle.mem_write(k, np.eye(dk), np.eye(dk), np.zeros((dk, P)), z0, nu, eps)
    np.testing.assert_array_equal(z, z0)


def test_orthogonal_keys_retrieved_independently():
    """Keys whose DPFP features have disjoint support are stored and read back
    without interference (up to the eps factor)."""
    dk, nu, eps = 2, 1, 1e-5
    k = np.array([[1.0, 0.5], [-1.0, -0.5]])      # r = (1,.5,0,0) and (0,0,1,.5)
    P = 2 * dk * nu
    wv = np.array([[2.0, 0.0], [0.0, -3.0]])
    A, z = oracle.mem_write(k, np.eye(dk), wv, np.zeros((dk, P)), np.zeros(P), nu, eps)
    phis = oracle.dpfp(k, nu)
    assert phis[0] @ phis[1] == 0.0
    r = oracle.mem_read(k, np.eye(dk), A, z, nu, eps)
    for j in range(2):
        n2 = phis[j] @ phis[j]
        np.testing.assert_allclose(r[j], (wv @ k[j]) * n2 / (n2 + eps), rtol=1e-12)


def test_gated_write_with_zero_gate_vector_halves_the_write_of_A():
    """w_beta = 0 gives beta = 1/2 for every row: into A = 0, z = 0 one row
    writes A = v phi^T / 2, while z (gamma = 1) is not gated: z = phi."""
    dk, nu, eps = 3, 2, 1e-5
    k = np.array([[0.7, -0.4, 1.1]])
    P = 2 * dk * nu
    A, z = oracle.mem_write(k, np.eye(dk), np.eye(dk), np.zeros((dk, P)), np.zeros(P), nu, eps,
                            w_beta=np.zeros(dk))
    phi = oracle.dpfp(k[0], nu)
    np.testing.assert_allclose(A, 0.5 * np.outer(k[0], phi), rtol=0, atol=1e-15)
    np.testing.assert_allclose(z, phi, rtol=0, atol=1e-15)


def test_gated_write_saturates_to_the_plain_write():
    """A gate vector that makes w_beta . m very large gives beta = 1 (the
    plain write); very negative gives beta = 0 (A unchanged, z still written)."""
    dk, nu, eps = 2, 2, 1e-5
    k = np.array([[0.3, -0.9]])
    P = 2 * dk * nu
    A0 = 0.1 * np.arange(dk * P, dtype=float).reshape(dk, P)
    z0 = np.abs(np.sin(np.arange(P, dtype=float)))
    plain = oracle.mem_write(k, np.eye(dk), np.eye(dk), A0, z0, nu, eps)
    hi = oracle.mem_write(k, np.eye(dk), np.eye(dk), A0, z0, nu, eps, w_beta=np.array([1e3, -1e3]))
    lo = oracle.mem_write(k, np.eye(dk), np.eye(dk), A0, z0, nu, eps, w_beta=np.array([-1e3, 1e3]))
    np.testing.assert_allclose(hi[0], plain[0], rtol=1e-14)
    np.testing.assert_array_equal(lo[0], A0)
    np.testing.assert_allclose(lo[1], plain[1], rtol=1e-14)


def test_unclamped_gamma_goes_negative():
    """With z = 2 phi(k), gamma = 1 - 2|phi|^2/(|phi|^2+eps) ~ -1: unclamped,
    z moves back to ~phi (clamped it stays, test_gamma_clamped_at_zero)."""
    dk, nu, eps = 2, 2, 1e-5
    k = np.array([[0.3, -0.9]])
    P = 2 * dk * nu
    phi = oracle.dpfp(k[0], nu)
    z0 = 2 * phi
    n2 = phi @ phi
    _, z = oracle.mem_write(k, np.eye(dk), np.eye(dk), np.zeros((dk, P)), z0, nu, eps, clamp_gamma=False)
    np.testing.assert_allclose(z, z0 + (1.0 - 2 * n2 / (n2 + eps)) * phi, rtol=1e-13)
    np.testing.assert_allclose(z, phi, rtol=4 * eps / n2)     # z0 - phi up to the eps terms


def test_read_of_empty_state_is_zero():
    x = RNG.standard_normal((5, 8))
    r = oracle.mem_read(x, RNG.standard_normal((2, 8)), np.zeros((8, 8)), np.zeros(8), 2, 1e-5)
    assert not r.any()


# --------------------------------------------------------------------------- layer parts

def test_rmsnorm_unit_rms_and_constant_row():
    x = RNG.standard_normal((4, 64)) * 7.0
    y = oracle.rms_norm(x, np.ones(64), 1e-12)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-10)
    c, eps = 0.3, 1e-5
    g = RNG.standard_normal(16)
    np.testing.assert_allclose(oracle.rms_norm(np.full((1, 16), c), g, eps)[0],
                               c / math.sqrt(c * c + eps) * g, rtol=1e-14)


def test_rope_identity_at_zero_norm_preserving_and_relative():
    hd, T, theta = 16, 9, 500000.0
    cos, sin = oracle.rope_cos_sin(T, hd, theta)
    x = RNG.standard_normal((T, 3, hd))
    y = oracle.apply_rope(x, cos, sin)
    np.testing.assert_allclose(y[0], x[0], rtol=0, atol=0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    # <R_p q, R_p' k> depends on p - p' only
    q, k = RNG.standard_normal(hd), RNG.standard_normal(hd)
    qs = oracle.apply_rope(np.tile(q, (T, 1, 1)), cos, sin)[:, 0]
    ks = oracle.apply_rope(np.tile(k, (T, 1, 1)), cos, sin)[:, 0]
    np.testing.assert_allclose(qs[5] @ ks[2], qs[6] @ ks[3], rtol=1e-12)
    np.testing.assert_allclose(qs[8] @ ks[4], qs[4] @ ks[0], rtol=1e-12)


def test_rope_matches_complex_rotation_and_inv_freq():
    """Rotate-half RoPE is multiplication of x_j + i x_{j+hd/2} by exp(i p theta^(-2j/hd))."""
    hd, T, theta = 8, 5, 10000.0
    cos, sin = oracle.rope_cos_sin(T, hd, theta)
    x = RNG.standard_normal((T, 1, hd))
    y = oracle.apply_rope(x, cos, sin)
    for p in range(T):
        for j in range(hd // 2):
            c = complex(x[p, 0, j], x[p, 0, j + hd // 2]) * np.exp(1j * p * theta ** (-2 * j / hd))
            assert abs(y[p, 0, j] - c.real) < 1e-12 and abs(y[p, 0, j + hd // 2] - c.imag) < 1e-12


def test_attention_closed_forms():
    T, H, hd = 6, 2, 4
    v = RNG.standard_normal((T, H, hd))
    k = RNG.standard_normal((T, H, hd))
    # one row: softmax of one score is 1
    out = oracle.causal_attention(RNG.standard_normal((1, H, hd)), k[:1], v[:1])
    np.testing.assert_allclose(out, v[:1], rtol=1e-15)
    # zero queries: uniform weights over the causal prefix
    out = oracle.causal_attention(np.zeros((T, H, hd)), k, v)
    for t in range(T):
        np.testing.assert_allclose(out[t], v[:t + 1].mean(axis=0), rtol=1e-13)
    # causality: changing rows > t0 leaves rows <= t0 unchanged
    q = RNG.standard_normal((T, H, hd))
    a = oracle.causal_attention(q, k, v)
    k2, v2 = k.copy(), v.copy()
    k2[4:] += 1.0
    v2[4:] -= 2.0
    b = oracle.causal_attention(q, k2, v2)
    np.testing.assert_array_equal(a[:4], b[:4])
    assert not np.allclose(a[4:], b[4:])


def test_gqa_equals_mha_with_repeated_kv_heads():
    """Query head h reads kv head floor(h KV / H): contiguous groups."""
    T, H, KV, hd = 5, 4, 2, 4
    q = RNG.standard_normal((T, H, hd))
    k = RNG.standard_normal((T, KV, hd))
    v = RNG.standard_normal((T, KV, hd))
    ref = oracle.causal_attention(q, np.repeat(k, H // KV, axis=1), np.repeat(v, H // KV, axis=1))
    np.testing.assert_allclose(oracle.causal_attention(q, k, v), ref, rtol=1e-14)


def test_silu_values():
    np.testing.assert_allclose(oracle.silu(np.array([0.0, 1.0, -1.0, 30.0])),
                               [0.0, 0.7310585786300049, -0.2689414213699951, 30.0], rtol=1e-12)


# --------------------------------------------------------------------------- whole model

def test_oracle_matches_pure_python_bruteforce():
    cfg = _micro()
    w = _micro_weights(cfg)
    emb = RNG.standard_normal((cfg.n_segments * cfg.seg_len, cfg.d_model))
    h, A, z = oracle.forward(cfg, w, emb)
    hn, An, zn = naive_armt.forward(cfg, w, emb)
    np.testing.assert_allclose(h, np.array(hn), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(A, np.array(An), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(z, np.array(zn), rtol=1e-11, atol=1e-13)
    assert np.abs(A).max() > 1e-3          # the memory path is exercised


def test_oracle_matches_bruteforce_gqa_and_odd_shapes():
    cfg = _micro(n_heads=4, n_kv_heads=2, head_dim=2, d_model=6, d_ffn=5, n_mem=3,
                 d_key=3, dpfp_nu=3, seg_len=2, n_segments=4, n_layers=3)
    w = _micro_weights(cfg, seed=11)
    emb = RNG.standard_normal((cfg.n_segments * cfg.seg_len, cfg.d_model))
    h, A, z = oracle.forward(cfg, w, emb)
    hn, An, zn = naive_armt.forward(cfg, w, emb)
    np.testing.assert_allclose(h, np.array(hn), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(A, np.array(An), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(z, np.array(zn), rtol=1e-11, atol=1e-13)


@pytest.mark.parametrize("gate,clamp", [(True, True), (False, False), (True, False)])
def test_oracle_variants_match_pure_python_bruteforce(gate, clamp):
    cfg = _micro(write_gate=gate, gamma_clamp=clamp, n_segments=4)
    w = _micro_weights(cfg, seed=5)
    emb = RNG.standard_normal((cfg.n_segments * cfg.seg_len, cfg.d_model))
    h, A, z = oracle.forward(cfg, w, emb)
    hn, An, zn = naive_armt.forward(cfg, w, emb)
    np.testing.assert_allclose(h, np.array(hn), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(A, np.array(An), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(z, np.array(zn), rtol=1e-11, atol=1e-13)
    base = oracle.forward(_micro(n_segments=4), w, emb)
    assert not np.allclose(A, base[1])      # the variant changes the state


def test_oracle_initial_state_matches_pure_python_bruteforce():
    cfg = _micro()
    w = _micro_weights(cfg, seed=9)
    P = cfg.phi_dim
    rng = np.random.default_rng(2)
    A0 = 0.2 * rng.standard_normal((cfg.n_layers, cfg.d_model, P))
    z0 = np.abs(rng.standard_normal((cfg.n_layers, P)))
    emb = RNG.standard_normal((cfg.n_segments * cfg.seg_len, cfg.d_model))
    h, A, z = oracle.forward(cfg, w, emb, A0=A0, z0=z0)
    hn, An, zn = naive_armt.forward(cfg, w, emb, A0=A0, z0=z0)
    np.testing.assert_allclose(h, np.array(hn), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(A, np.array(An), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(z, np.array(zn), rtol=1e-11, atol=1e-13)


@pytest.mark.parametrize("name,split", [("tiny", 1), ("tiny", 3), ("small", 2)])
def test_streaming_in_two_calls_equals_one_call(name, split):
    """Resume: S1 segments, then the next S2 segments from the carried state,
    equal S1 + S2 segments in one call, bit for bit (the same operations in
    the same order)."""
    cfg = CONFIGS[name]
    S = 4 if name == "small" else cfg.n_segments
    T = cfg.seg_len
    w = make_weights(cfg)
    emb = make_embeddings(cfg, S)
    h, A, z = oracle.forward(cfg, w, emb)
    h1, A1, z1 = oracle.forward(cfg, w, emb[:split * T])
    h2, A2, z2 = oracle.forward(cfg, w, emb[split * T:], A0=A1, z0=z1)
    np.testing.assert_array_equal(np.concatenate([h1, h2]), h)
    np.testing.assert_array_equal(A2, A)
    np.testing.assert_array_equal(z2, z)


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_sequential_and_diagonal_orders_bitwise_equal(name):
    cfg = CONFIGS[name]
    S = 6 if name == "small" else cfg.n_segments
    w = make_weights(cfg)
    emb = make_embeddings(cfg, S)
    a = oracle.forward(cfg, w, emb)
    b = oracle.forward(cfg, w, emb, order=oracle.diagonal_order(S, cfg.n_layers))
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_order_violating_dependencies_is_refused():
    cfg = CONFIGS["tiny"]
    w = make_weights(cfg)
    emb = make_embeddings(cfg)
    bad = [(0, 0), (1, 0), (1, 1), (0, 1), (2, 0), (2, 1), (3, 0), (3, 1)]   # (1,1) before (0,1)
    with pytest.raises(ValueError):
        oracle.forward(cfg, w, emb, order=bad)


def test_prefix_invariance():
    cfg = CONFIGS["tiny"]
    w = make_weights(cfg)
    emb = make_embeddings(cfg)
    h, A, z = oracle.forward(cfg, w, emb)
    h2, _, _ = oracle.forward(cfg, w, emb[:2 * cfg.seg_len])
    np.testing.assert_array_equal(h[:2 * cfg.seg_len], h2)


def test_without_memory_segments_are_independent_llama_forwards():
    cfg = CONFIGS["tiny"]
    w = make_weights(cfg)
    emb = make_embeddings(cfg)
    h, A, z = oracle.forward(cfg, w, emb, memory=False)
    assert not A.any() and not z.any()
    T = cfg.seg_len
    for s in range(cfg.n_segments):
        hs, _, _ = oracle.forward(cfg, w, emb[s * T:(s + 1) * T], memory=False)
        np.testing.assert_array_equal(h[s * T:(s + 1) * T], hs)
    # with one segment, the memory read adds exactly 0: same as no memory
    h1, _, _ = oracle.forward(cfg, w, emb[:T])
    np.testing.assert_array_equal(h1, h[:T])


def test_memory_carries_information_across_segments():
    cfg = CONFIGS["tiny"]
    w = make_weights(cfg)
    emb = make_embeddings(cfg)
    h, _, _ = oracle.forward(cfg, w, emb)
    emb2 = emb.copy()
    emb2[:cfg.seg_len] += 1.0                  # change segment 0 only
    h2, _, _ = oracle.forward(cfg, w, emb2)
    T = cfg.seg_len
    assert not np.array_equal(h[T:], h2[T:])   # later segments see it through (A, z)


# --------------------------------------------------------------------------- planted mistakes

def _run_pins(monkeypatch, name, fn):
    monkeypatch.setattr(ao, name, fn)
    monkeypatch.setattr(oracle, name, fn, raising=False)


def _fails(test):
    try:
        test()
    except AssertionError:
        return True
    return False


def test_planted_roll_direction_is_caught(monkeypatch):
    def bad_dpfp(x, nu):
        r = np.concatenate([np.maximum(x, 0.0), np.maximum(-x, 0.0)], axis=-1)
        return np.concatenate([r * np.roll(r, -n, axis=-1) for n in range(1, nu + 1)], axis=-1)
    _run_pins(monkeypatch, "dpfp", bad_dpfp)
    assert _fails(test_dpfp_hand_values)


def test_planted_kv_head_mapping_is_caught(monkeypatch):
    def bad_attn(q, k, v):
        T, H, hd = q.shape
        KV = k.shape[1]
        out = np.empty_like(q)
        mask = np.triu(np.ones((T, T), dtype=bool), k=1)
        for h in range(H):
            g = h % KV
            sc = (q[:, h, :] @ k[:, g, :].T) / np.sqrt(hd)
            sc[mask] = -np.inf
            p = np.exp(sc - sc.max(axis=-1, keepdims=True))
            out[:, h, :] = (p / p.sum(axis=-1, keepdims=True)) @ v[:, g, :]
        return out
    _run_pins(monkeypatch, "causal_attention", bad_attn)
    assert _fails(test_gqa_equals_mha_with_repeated_kv_heads)
    assert _fails(test_oracle_matches_bruteforce_gqa_and_odd_shapes)


def test_planted_write_rows_are_caught(monkeypatch):
    orig = ao.node_forward

    def bad_node(x, w, l, A, z, cfg, memory=True):
        if memory:
            x = x + ao.mem_read(x, w["wq_mem"][l], A, z, cfg.dpfp_nu, cfg.mem_eps)
        x = ao.decoder_layer(x, w, l, cfg)
        if memory:   # wrong rows: the first M instead of the memory tokens
            m = ao.rms_norm(x[:cfg.n_mem], np.ones(x.shape[1]), cfg.rms_eps)
            A, z = ao.mem_write(m, w["wk_mem"][l], w["wv_mem"][l], A, z, cfg.dpfp_nu, cfg.mem_eps)
        return x, A, z
    monkeypatch.setattr(ao, "node_forward", bad_node)
    assert _fails(test_oracle_matches_pure_python_bruteforce)
    monkeypatch.setattr(ao, "node_forward", orig)


def test_planted_transposed_weight_is_caught(monkeypatch):
    orig = ao.decoder_layer

    def bad_layer(x, w, l, cfg):
        w2 = dict(w)
        w2["wo"] = np.swapaxes(w["wo"], 1, 2).copy()    # square at micro size
        return orig(x, w2, l, cfg)
    monkeypatch.setattr(ao, "decoder_layer", bad_layer)
    assert _fails(test_oracle_matches_pure_python_bruteforce)


def test_planted_gamma_sign_is_caught(monkeypatch):
    def bad_write(m, wk, wv, A, z, nu, eps, **kw):
        k = m @ wk.T
        v = m @ wv.T
        phi = ao.dpfp(k, nu)
        A, z = A.copy(), z.copy()
        for j in range(m.shape[0]):
            zphi = phi[j] @ z
            vbar = (A @ phi[j]) / (zphi + eps)
            gamma = min(max(1.0 + zphi / (phi[j] @ phi[j] + eps), 0.0), 1.0)
            A += np.outer(v[j] - vbar, phi[j])
            z += gamma * phi[j]
        return A, z
    _run_pins(monkeypatch, "mem_write", bad_write)
    assert _fails(test_rewrite_same_key_replaces_value)


def test_planted_batched_write_is_caught(monkeypatch):
    def batched_write(m, wk, wv, A, z, nu, eps, **kw):
        k = m @ wk.T
        v = m @ wv.T
        phi = ao.dpfp(k, nu)
        zphi = phi @ z
        vbar = (phi @ A.T) / (zphi + eps)[:, None]
        gamma = np.clip(1.0 - zphi / (np.sum(phi * phi, axis=-1) + eps), 0.0, 1.0)
        return A + (v - vbar).T @ phi, z + gamma @ phi
    _run_pins(monkeypatch, "mem_write", batched_write)
    assert _fails(test_write_rows_apply_one_after_another)
    assert _fails(test_oracle_matches_pure_python_bruteforce)


def test_planted_missing_write_norm_is_caught(monkeypatch):
    def node_no_norm(x, w, l, A, z, cfg, memory=True):
        if memory:
            x = x + ao.mem_read(x, w["wq_mem"][l], A, z, cfg.dpfp_nu, cfg.mem_eps)
        x = ao.decoder_layer(x, w, l, cfg)
        if memory:
            A, z = ao.mem_write(x[cfg.seg_len:], w["wk_mem"][l], w["wv_mem"][l], A, z, cfg.dpfp_nu, cfg.mem_eps)
        return x, A, z
    monkeypatch.setattr(ao, "node_forward", node_no_norm)
    assert _fails(test_oracle_matches_pure_python_bruteforce)


def test_planted_gate_on_z_is_caught(monkeypatch):
    """A gate that also scaled the z update would be a different reading:
    the brute force (gate on A only) catches it."""
    orig = ao.mem_write

    def gate_on_z(m, wk, wv, A, z, nu, eps, w_beta=None, clamp_gamma=True):
        A1, z1 = orig(m, wk, wv, A, z, nu, eps, w_beta=w_beta, clamp_gamma=clamp_gamma)
        if w_beta is None:
            return A1, z1
        return A1, z + ao.sigmoid(m @ w_beta).mean() * (z1 - z)
    _run_pins(monkeypatch, "mem_write", gate_on_z)
    assert _fails(lambda: test_oracle_variants_match_pure_python_bruteforce(True, True))


def test_planted_ignored_initial_state_is_caught(monkeypatch):
    orig = ao.forward

    def ignores_state(cfg, weights, emb, order=None, memory=True, A0=None, z0=None):
        return orig(cfg, weights, emb, order=order, memory=memory)
    monkeypatch.setattr(ao, "forward", ignores_state)
    monkeypatch.setattr(oracle, "forward", ignores_state)
    assert _fails(lambda: test_streaming_in_two_calls_equals_one_call("tiny", 1))


def test_no_memory_tokens_is_the_memoryless_forward():
    """n_mem = 0: no memory rows are written, so the state stays 0 and every
    read adds 0; the forward equals the memory=False hook (independent
    causal decoder forwards per segment) bit for bit."""
    cfg = CONFIGS["tiny"].with_(n_mem=0, n_segments=3)
    w = make_weights(cfg)
    emb = make_embeddings(cfg, 3)
    a = oracle.forward(cfg, w, emb)
    b = oracle.forward(cfg, w, emb, memory=False)
    np.testing.assert_array_equal(a[0], b[0])
    assert not a[1].any() and not a[2].any()
