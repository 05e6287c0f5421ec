"""The layer-pipelined forward's driver (recurrent_memory_transformer_diag_b200/
pipeline.py) on the CPU.

* Its per-wave hand-off plan against brute force over the dependency graph:
  a stage receives exactly the rows of the edges (s, first - 1) -> (s, first)
  that enter its block, in the wave of the receiving node, and sends exactly
  the rows of the edges that leave it, in the wave of the sending node.
* Two and three gloo ranks on the CPU, each computing its layer block's nodes
  with the fp64 oracle's node function: the last rank's hidden states and
  every rank's A_l, z_l equal the oracle's single-process forward bit for bit
  (the same fp64 operations on the same inputs).  The oracle is the stage
  compute only in this test; on a GPU the stage compute is armt_stage_wave.
"""
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_layer_blocks_cover_the_layers_evenly():
    from recurrent_memory_transformer_diag_b200.pipeline import layer_blocks
    for L in range(1, 20):
        for n in range(1, L + 1):
            b = layer_blocks(L, n)
            assert len(b) == n and b[0][0] == 0
            assert all(b[g][0] + b[g][1] == b[g + 1][0] for g in range(n - 1))
            assert b[-1][0] + b[-1][1] == L
            sizes = [c for _, c in b]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    with pytest.raises(ValueError):
        layer_blocks(3, 4)


def test_wave_io_is_the_block_crossing_edges():
    from recurrent_memory_transformer_diag_b200.pipeline import layer_blocks, wave_io
    for S in range(1, 7):
        for L in range(1, 8):
            for n in range(1, L + 1):
                for off, cnt in layer_blocks(L, n):
                    first, last = off, off + cnt - 1
                    # brute force: every edge (s, l-1) -> (s, l) of the layer grid
                    want_recv = {s + first for s in range(S)} if first > 0 else set()
                    want_send = {s + last for s in range(S)} if last < L - 1 else set()
                    got_recv = {i for i in range(S + L - 1) if wave_io(i, S, off, cnt, L)[0]}
                    got_send = {i for i in range(S + L - 1) if wave_io(i, S, off, cnt, L)[1]}
                    assert got_recv == want_recv and got_send == want_send, (S, L, off, cnt)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, S, L, out):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from recurrent_memory_transformer_diag_b200.inputs import CONFIGS, make_embeddings, make_weights
    from recurrent_memory_transformer_diag_b200.pipeline import layer_blocks, run_stage
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        cfg = CONFIGS["tiny"].with_(n_layers=L, n_segments=S)
        w = {k: np.asarray(v, dtype=np.float64) for k, v in make_weights(cfg).items()}
        emb = np.asarray(make_embeddings(cfg, S), dtype=np.float64)
        T, d, P = cfg.seg_len, cfg.d_model, cfg.phi_dim
        off, cnt = layer_blocks(L, world)[rank]
        A = np.zeros((cnt, d, P))
        z = np.zeros((cnt, P))
        cur = {}
        hidden = np.zeros((S * T, d))
        in_rows = torch.zeros(T + cfg.n_mem, d, dtype=torch.float64)
        out_rows = torch.zeros(T + cfg.n_mem, d, dtype=torch.float64)

        def stage_wave(i, inb, outb):
            for j in range(cnt):
                s, l = i - off - j, off + j
                if not 0 <= s < S:
                    continue
                if j > 0:
                    x = cur.pop(s)
                elif off == 0:
                    x = np.concatenate([emb[s * T:(s + 1) * T], w["mem_emb"]], axis=0)
                else:
                    x = inb.numpy().copy()
                x, A[j], z[j] = oracle.node_forward(x, w, l, A[j], z[j], cfg)
                if j < cnt - 1:
                    cur[s] = x
                elif l == L - 1:
                    hidden[s * T:(s + 1) * T] = x[:T]
                else:
                    outb.copy_(torch.from_numpy(x))

        run_stage(stage_wave, S, L, off, cnt, rank, in_rows, out_rows)
        out.put((rank, off, A, z, hidden if off + cnt == L else None))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,L,S", [(2, 4, 5), (3, 4, 3)])
def test_gloo_pipeline_equals_single_process_forward(world, L, S):
    import multiprocessing as mp
    sys.path.insert(0, ROOT)
    import oracle
    from recurrent_memory_transformer_diag_b200.inputs import CONFIGS, make_embeddings, make_weights
    cfg = CONFIGS["tiny"].with_(n_layers=L, n_segments=S)
    ref_h, ref_A, ref_z = oracle.forward(cfg, make_weights(cfg), make_embeddings(cfg, S))
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, S, L, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in range(world)), key=lambda r: r[0])
    for p in procs:
        p.join(60)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    for rank, off, A, z, hidden in res:
        np.testing.assert_array_equal(A, ref_A[off:off + A.shape[0]])
        np.testing.assert_array_equal(z, ref_z[off:off + z.shape[0]])
    np.testing.assert_array_equal(res[-1][4], ref_h)
