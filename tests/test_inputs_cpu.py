"""The seeded input recipe shared by the oracle and the CUDA path: fixed
shapes, determinism, the prefix property the large parity tests rely on, and
bf16 workloads feeding both sides values already rounded to bf16."""
import numpy as np
import pytest
import torch

from recurrent_memory_transformer_diag_b200.inputs import CONFIGS, make_embeddings, make_weights


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_weights_shapes_and_determinism(name):
    cfg = CONFIGS[name]
    w1, w2 = make_weights(cfg), make_weights(cfg)
    shapes = cfg.weight_shapes()
    assert set(w1) == set(shapes)
    for k, a in w1.items():
        assert a.shape == tuple(shapes[k]) and a.dtype == np.float32
        np.testing.assert_array_equal(a, w2[k])
    np.testing.assert_array_equal(w1["attn_norm"], 1.0)   # gains are ones
    np.testing.assert_array_equal(w1["mlp_norm"], 1.0)
    assert not np.array_equal(w1["wq"], make_weights(cfg, seed=7)["wq"])
    assert 0.015 < float(w1["wq"].std()) < 0.025          # N(0, 0.02) draws


def test_embedding_prefix_property():
    cfg = CONFIGS["small"]
    full = make_embeddings(cfg)
    two = make_embeddings(cfg, 2)
    assert full.shape == (cfg.n_segments * cfg.seg_len, cfg.d_model)
    np.testing.assert_array_equal(two, full[: 2 * cfg.seg_len])
    assert 0.9 < float(full.std()) < 1.1


def test_bf16_workloads_are_bf16_representable():
    cfg = CONFIGS["small"]
    assert cfg.dtype == "bf16"
    for a in (make_weights(cfg)["w_up"], make_embeddings(cfg, 1)):
        t = torch.from_numpy(a)
        np.testing.assert_array_equal(t.to(torch.bfloat16).to(torch.float32).numpy(), a)


def test_optional_gains_are_drawn_around_one():
    cfg = CONFIGS["small"]
    w = make_weights(cfg, gain_std=0.1)
    for name in ("attn_norm", "mlp_norm"):
        g = w[name]
        assert 0.07 < float(g.std()) < 0.13 and abs(float(g.mean()) - 1.0) < 0.02
    assert not np.array_equal(w["attn_norm"], w["mlp_norm"])
    base = make_weights(cfg)
    np.testing.assert_array_equal(w["wq"], base["wq"])     # only the gains change
