"""CPU oracle for the ARMT diagonal-batching forward: TEST INFRASTRUCTURE.

Plain, slow, fp64 restatement of what the hot path computes, written from
the pages' definitions (see each module's header).  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import it; the product path never does.

Every function here is pinned by ``tests/test_oracle_*.py`` to something
other than itself (hand-computed values in ``tests/golden/``, closed forms,
invariants, an independent brute-force restatement on tiny inputs).
"""
from .armt_oracle import (apply_rope, causal_attention, decoder_layer, diagonal_order,  # noqa: F401
                          dpfp, forward, mem_read, mem_write, node_forward, rms_norm,
                          rope_cos_sin, silu)
from .schedule import (check_schedule, diagonal_waves, earliest_groups,  # noqa: F401
                       prmt_dependencies, rmt_dependencies, sequential_order)
