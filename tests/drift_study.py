"""How the ARMT recurrence amplifies small per-node errors (not collected by
pytest; about 3 minutes of host time with the defaults).

Runs the fp64 oracle twice on the 1B layer shapes (segments shortened to
--seg-len tokens to keep it cheap): once exactly, once with unbiased relative
noise of size --noise multiplied into every layer's output before the memory
write (x <- x (1 + noise N(0, 1)), independently per element), a stand-in for
the rounding of a 16-bit-activation implementation (fp16 rounding is at most
2^-11 relative, 2^-12 on average).  Prints the relative L2 error of every
segment's hidden states and of every layer's A and z.  With noise 5e-4 the
error grows from 2.9e-3 (segment 0) to 1.6e-2 (segment 17) and A reaches
1-2.5 %: the delta-rule write turns small errors in the memory rows into
larger errors in A, which the next segments read back.

    python tests/drift_study.py [--seg-len 64] [--segments 18] [--noise 5e-4]
"""
import argparse
import os
import sys
import time

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--seg-len", type=int, default=64)
    ap.add_argument("--segments", type=int, default=18)
    ap.add_argument("--noise", type=float, default=5e-4)
    ap.add_argument("--seed", type=int, default=0)
    a = ap.parse_args()
    import oracle
    from oracle import armt_oracle as ao
    from recurrent_memory_transformer_diag_b200.inputs import CONFIGS, make_embeddings, make_weights
    S, T = a.segments, a.seg_len
    cfg = CONFIGS["1b"].with_(seg_len=T, n_segments=S)
    w = make_weights(cfg)
    emb = make_embeddings(cfg, S)
    t0 = time.time()
    ref = oracle.forward(cfg, w, emb)
    rng = np.random.default_rng(a.seed)
    exact_layer = ao.decoder_layer

    def noisy_layer(x, w_, l, cfg_):
        x = exact_layer(x, w_, l, cfg_)
        return x * (1.0 + a.noise * rng.standard_normal(x.shape))

    ao.decoder_layer = noisy_layer
    try:
        got = oracle.forward(cfg, w, emb)
    finally:
        ao.decoder_layer = exact_layer

    def rel(x, y):
        return float(np.linalg.norm(x - y) / np.linalg.norm(y))

    print(f"1B layers, {S} segments of {T} tokens, noise {a.noise} per layer output ({time.time() - t0:.0f} s)")
    print("hidden per segment:", " ".join(f"{rel(got[0][s * T:(s + 1) * T], ref[0][s * T:(s + 1) * T]):.2e}"
                                          for s in range(S)))
    print("A per layer:", " ".join(f"{rel(got[1][l], ref[1][l]):.2e}" for l in range(cfg.n_layers)))
    print("z per layer:", " ".join(f"{rel(got[2][l], ref[2][l]):.2e}" for l in range(cfg.n_layers)))


if __name__ == "__main__":
    main()
