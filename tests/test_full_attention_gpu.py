"""No associative memory (n_mem = 0): each segment is a plain causal decoder
forward, and one segment of N tokens is the full-attention decoder over N
tokens, run on the same grouped GEMMs and the same tensor-core attention.
This is the baseline the pages compare ARMT with (Pith review, Figure 1
caption: full-attention Llama-3.2-1B at 131072 tokens).

* Against the oracle (whose memory read of a zero state adds exactly 0 and
  whose write of zero rows changes nothing): tiny fp32 (<= 1e-5), small and
  the 1B and 3B layer shapes over 2048 tokens in bf16 mode (<= 1e-2).
* The 131072-token 1B forward, the benchmarked launch: its first 2048 rows
  equal the 2048-token run bit for bit (each query tile attends to the same
  keys in the same order, each GEMM tile sees the same rows), all finite.
"""
import numpy as np
import pytest

import oracle
from recurrent_memory_transformer_diag_b200.inputs import CONFIGS, make_embeddings, make_weights

from .gpu_util import rel_l2, run_gpu

pytestmark = pytest.mark.gpu


def _no_memory(name, T, S=1):
    return CONFIGS[name].with_(n_mem=0, seg_len=T, n_segments=S)


@pytest.mark.parametrize("name,T,S,tol", [("tiny", 16, 3, 1e-5), ("small", 512, 2, 1e-2),
                                          ("1b", 2048, 1, 1e-2), ("3b", 2048, 1, 1e-2)])
def test_no_memory_matches_oracle(name, T, S, tol):
    cfg = _no_memory(name, T, S)
    w = make_weights(cfg)
    emb = make_embeddings(cfg, S)
    h, A, z = oracle.forward(cfg, w, emb)
    assert not A.any() and not z.any()
    got = run_gpu(cfg, w, emb, S)
    for s in range(S):
        err = rel_l2(got[0][s * T:(s + 1) * T], h[s * T:(s + 1) * T])
        print(f"\n{name} no memory, T={T}, segment {s}: rel-L2 {err:.3e}")
        assert err <= tol
    assert not got[1].any() and not got[2].any()


def test_full_attention_131072_tokens_prefix_and_finite():
    import torch
    from recurrent_memory_transformer_diag_b200 import Armt
    N, n0 = 131072, 2048
    cfg = _no_memory("1b", N)
    w = make_weights(cfg)
    emb = make_embeddings(cfg, 1)
    m = Armt(cfg, max_segments=1)
    m.load_weights(w)
    big = run_gpu(cfg, w, emb, 1, model=m)[0]
    m.close()
    assert np.isfinite(big).all()
    c0 = _no_memory("1b", n0)
    small = run_gpu(c0, w, emb[:n0], 1)[0]
    np.testing.assert_array_equal(big[:n0], small)
    del torch
