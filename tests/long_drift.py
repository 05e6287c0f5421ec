"""Drift of the full-length 1B forward against the fp64 oracle.

Not collected by pytest (the oracle needs about an hour of host time for the
128 segments).  Three steps, each writing an .npz:

    python tests/long_drift.py oracle  --out ORACLE.npz          # host, fp64 oracle
    python tests/long_drift.py gpu     --out GPU.npz [--dtype bf16|fp32] [--ref ORACLE.npz]   # B200
    python tests/long_drift.py compare ORACLE.npz GPU.npz [GPU2.npz ...]

Both sides use the seeded inputs of the 131072-token workload (128 segments
of 1024 tokens + 16 memory tokens, L = 16, d = 2048).  Stored per segment:
rows 0, 64, ..., 960 of the final hidden states (a fixed sample of every
segment); at the end A and z of every layer (fp32; the GPU side's A as an
fp16 copy in bf16 mode, whose 2^-11 rounding is far below the compared
errors).  The oracle step saves a resumable fp64 state every 8 segments.  `compare` prints, per
segment, the relative L2 error of the sampled rows and, per layer, that of
A and z.
"""
import argparse
import json
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

ROWS = np.arange(0, 1024, 64)


def _cfg(dtype="bf16"):
    from recurrent_memory_transformer_diag_b200.inputs import CONFIGS
    return CONFIGS["1b"].with_(dtype=dtype)


def run_oracle(out, S):
    import oracle
    from recurrent_memory_transformer_diag_b200.inputs import make_embeddings, make_weights
    cfg = _cfg()
    w = {k: np.asarray(v, dtype=np.float64) for k, v in make_weights(cfg).items()}   # converted once
    emb = make_embeddings(cfg, S)
    T, L, d, P = cfg.seg_len, cfg.n_layers, cfg.d_model, cfg.phi_dim
    # the recurrence one segment at a time (carrying the state), so progress
    # can be saved and resumed; identical to one call over all segments
    # (the streaming identity is pinned in tests/test_oracle_pins.py)
    ckpt = out + ".state.npz"
    A = np.zeros((L, d, P))
    z = np.zeros((L, P))
    rows = np.zeros((S, len(ROWS), d), dtype=np.float32)
    start = 0
    if os.path.exists(ckpt):
        c = np.load(ckpt)
        start, A, z = int(c["segments"]), c["A"], c["z"]
        rows[:start] = c["rows"][:start]
    t0 = time.time()
    for s in range(start, S):
        h, A, z = oracle.forward(cfg, w, emb[s * T:(s + 1) * T], A0=A, z0=z)
        rows[s] = h[ROWS]
        print(f"segment {s} done, {time.time() - t0:.0f} s", flush=True)
        if s % 8 == 7 or s == S - 1:
            np.savez(ckpt, rows=rows[:s + 1], A=A, z=z, segments=s + 1)
            np.savez(out, rows=rows[:s + 1], A=A.astype(np.float32), z=z.astype(np.float32), segments=s + 1)


def run_gpu(out, S, dtype, ref=None):
    import torch
    from recurrent_memory_transformer_diag_b200 import Armt
    from recurrent_memory_transformer_diag_b200.inputs import make_embeddings, make_weights
    cfg_w = _cfg()                       # bf16-valued weights and inputs for both modes
    cfg = _cfg(dtype)
    w = make_weights(cfg_w)
    emb = make_embeddings(cfg_w, S)
    T, L, d, P = cfg.seg_len, cfg.n_layers, cfg.d_model, cfg.phi_dim
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    m = Armt(cfg, max_segments=S)
    m.load_weights(w)
    e = torch.from_numpy(emb).cuda().to(dt)
    o = torch.empty(S * T, d, dtype=dt, device="cuda")
    A = torch.empty(L, d, P, device="cuda")
    z = torch.empty(L, P, device="cuda")
    t0 = time.time()
    m.forward(e, S, T, o, A, z)
    m.device_status()
    torch.cuda.synchronize()
    secs = time.time() - t0
    idx = torch.tensor([s * T + r for s in range(S) for r in ROWS], device="cuda")
    rows = o.index_select(0, idx).float().reshape(S, len(ROWS), d).cpu().numpy()
    A_keep = A.half() if dtype == "bf16" else A
    np.savez(out, rows=rows, A=A_keep.cpu().numpy(), z=z.cpu().numpy(), segments=S, seconds=secs)
    m.close()
    print(f"{dtype}: {S} segments in {secs:.2f} s -> {out}")
    if ref:   # compare right here and keep only the small summary
        summary = compare(ref, [out])
        os.remove(out)
        with open(out.replace(".npz", ".json"), "w") as f:
            json.dump(summary, f)


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def compare(ref_path, paths):
    ref = np.load(ref_path)
    S = int(ref["segments"])
    out = {}
    for p in paths:
        g = np.load(p)
        n = min(S, int(g["segments"]))
        seg = [rel(g["rows"][s], ref["rows"][s]) for s in range(n)]
        res = {"segments": n, "hidden_per_segment": seg}
        if n == int(ref["segments"]) and n == int(g["segments"]):
            res["A_per_layer"] = [rel(g["A"][l], ref["A"][l]) for l in range(ref["A"].shape[0])]
            res["z_per_layer"] = [rel(g["z"][l], ref["z"][l]) for l in range(ref["z"].shape[0])]
        out[os.path.basename(p)] = res
        print(f"{p}: {n} segments")
        for s in range(0, n, 8):
            print("  seg %3d..%3d: " % (s, min(n, s + 8) - 1) + " ".join(f"{v:.2e}" for v in seg[s:s + 8]))
        if "A_per_layer" in res:
            print("  A per layer: " + " ".join(f"{v:.2e}" for v in res["A_per_layer"]))
            print("  z per layer: " + " ".join(f"{v:.2e}" for v in res["z_per_layer"]))
    print(json.dumps({k: {"worst_segment": max(v["hidden_per_segment"]),
                          "worst_A": max(v.get("A_per_layer", [0])),
                          "worst_z": max(v.get("z_per_layer", [0]))} for k, v in out.items()}))
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("mode", choices=["oracle", "gpu", "compare"])
    ap.add_argument("paths", nargs="*")
    ap.add_argument("--out")
    ap.add_argument("--segments", type=int, default=128)
    ap.add_argument("--dtype", default="bf16", choices=["bf16", "fp32"])
    ap.add_argument("--ref", default=None, help="gpu: oracle .npz to compare with on the spot")
    a = ap.parse_args()
    if a.mode == "oracle":
        run_oracle(a.out, a.segments)
    elif a.mode == "gpu":
        run_gpu(a.out, a.segments, a.dtype, a.ref)
    else:
        compare(a.paths[0], a.paths[1:])


if __name__ == "__main__":
    main()
