"""The memory write of each wave runs on a second stream and overlaps the
next wave's first kernels (tensor-core path).  The overlap changes only when
kernels run, never what they compute: with it turned off in a child process
(ARMT_OVERLAP_WRITE=0) the small forward (both schedules, graph-captured and
directly launched, and the overlapped host-buffer forward) and the 1B forward
over 18 segments give the same bits."""
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import sys, numpy as np, torch
    sys.path.insert(0, "tests")
    from gpu_util import run_gpu
    from recurrent_memory_transformer_diag_b200 import Armt
    from recurrent_memory_transformer_diag_b200.inputs import CONFIGS, make_embeddings, make_weights
    out = {}
    for name, S, combos in (("small", 16, [("diagonal", True), ("diagonal", False), ("sequential", True),
                                           ("sequential", False)]),
                            ("1b", 18, [("diagonal", True), ("sequential", False)])):
        cfg = CONFIGS[name]
        w = make_weights(cfg)
        emb = make_embeddings(cfg, S)
        for sched, graph in combos:
            if True:
                h, A, z = run_gpu(cfg, w, emb, S, schedule=sched, graph=graph)
                out[f"{name}_{sched}_{int(graph)}_h"] = h
                out[f"{name}_{sched}_{int(graph)}_A"] = A
                out[f"{name}_{sched}_{int(graph)}_z"] = z
    cfg = CONFIGS["small"]
    m = Armt(cfg)
    m.load_weights(make_weights(cfg))
    dt = torch.bfloat16
    he = torch.from_numpy(make_embeddings(cfg)).to(dt).pin_memory()
    ho = torch.empty(cfg.n_tokens, cfg.d_model, dtype=dt).pin_memory()
    hA = torch.empty(cfg.n_layers, cfg.d_model, cfg.phi_dim).pin_memory()
    hz = torch.empty(cfg.n_layers, cfg.phi_dim).pin_memory()
    m.forward_host(he, cfg.n_segments, cfg.seg_len, ho, hA, hz)
    out["host_h"] = ho.float().numpy(); out["host_A"] = hA.numpy(); out["host_z"] = hz.numpy()
    np.savez(sys.argv[1], **out)
    print("OVERLAP_CHILD_OK")
""")


def _run(tmp_path, overlap):
    env = dict(os.environ, ARMT_OVERLAP_WRITE="1" if overlap else "0")
    path = str(tmp_path / f"ov{int(overlap)}.npz")
    r = subprocess.run([sys.executable, "-c", CHILD, path], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0 and "OVERLAP_CHILD_OK" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
    return np.load(path)


def test_write_overlap_changes_no_bits(tmp_path):
    a = _run(tmp_path, True)
    b = _run(tmp_path, False)
    assert set(a.files) == set(b.files)
    for k in a.files:
        np.testing.assert_array_equal(a[k], b[k], err_msg=k)
