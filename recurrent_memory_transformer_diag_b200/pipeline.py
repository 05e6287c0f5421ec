"""Layer-pipelined forward over several GPUs: one stage (a contiguous block of
layers) per rank, one segment's residual rows handed to the next stage per
wave.

Wave i of the diagonal schedule holds the nodes (s, l) with s + l = i (Pith
review of arXiv 2506.05229, "What carries the argument": the wave is a
wavefront over the layer grid).  Cut the layers into contiguous blocks, one
per rank, and every rank can run its part of wave i at the same time: the
only dependency that crosses ranks is node (s, first) of a block on node
(s, first - 1) of the block before it, computed one wave earlier.  A layer's
memory state A_l, z_l never leaves its rank.  Per wave a rank therefore
receives at most one [T', d] block of rows from its predecessor and sends at
most one to its successor, point to point (``torch.distributed`` send / recv;
NCCL over NVLink between GPUs).

The compute of a stage is a callable ``stage_wave(wave, in_rows, out_rows)``;
on a GPU it is the library's ``armt_stage_wave`` (``gpu_stage`` below).  This
module decides, per wave, what is received, computed and sent; it does no
arithmetic of the model.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Tuple


def layer_blocks(total_layers: int, stages: int) -> List[Tuple[int, int]]:
    """Contiguous blocks (offset, n_layers) covering 0 .. total_layers - 1,
    sizes differing by at most one (earlier stages take the extra layers)."""
    if stages < 1 or stages > total_layers:
        raise ValueError("need 1 <= stages <= total_layers")
    base, extra = divmod(total_layers, stages)
    blocks, off = [], 0
    for g in range(stages):
        n = base + (1 if g < extra else 0)
        blocks.append((off, n))
        off += n
    return blocks


def wave_io(wave: int, n_segments: int, offset: int, n_layers: int, total_layers: int) -> Tuple[bool, bool]:
    """(receive, send) for a stage holding layers offset .. offset + n_layers - 1
    in global wave `wave`: it receives the rows of segment wave - offset (the
    previous block's output, sent in the wave before) when that segment exists
    and the block is not the first, and sends those of segment
    wave - (offset + n_layers - 1) when that segment exists and the block is
    not the last."""
    first, last = offset, offset + n_layers - 1
    recv = first > 0 and 0 <= wave - first < n_segments
    send = last < total_layers - 1 and 0 <= wave - last < n_segments
    return recv, send


def run_stage(stage_wave: Callable[[int, Optional[object], Optional[object]], None], n_segments: int,
              total_layers: int, offset: int, n_layers: int, rank: int, in_rows, out_rows,
              group=None) -> None:
    """Run every global wave of this rank's stage (rank r holds the r-th block
    and talks to ranks r - 1 and r + 1).  in_rows / out_rows: this rank's
    [T', d] hand-off buffers (on the GPU for NCCL, on the host for gloo).
    Receives and sends are in wave order on both sides of each rank pair, and
    rows only flow to the next rank, so the exchange cannot deadlock."""
    import torch.distributed as dist
    for i in range(n_segments + total_layers - 1):
        recv, send = wave_io(i, n_segments, offset, n_layers, total_layers)
        if recv:
            dist.recv(in_rows, src=rank - 1, group=group)
        stage_wave(i, in_rows if recv else None, out_rows if send else None)
        if send:
            dist.send(out_rows, dst=rank + 1, group=group)


def gpu_stage(model, n_segments: int, seg_len: int, offset: int, total_layers: int, emb, out_hidden, A, z,
              carry_state: bool = False):
    """The stage compute of a GPU rank: ``Armt.stage_wave`` (armt_stage_wave)
    on the current stream for a context holding this rank's layer block."""
    def stage_wave(i, in_rows, out_rows):
        model.stage_wave(n_segments, seg_len, i, offset, total_layers, emb, in_rows, out_rows, out_hidden, A, z,
                         carry_state=carry_state)
    return stage_wave
