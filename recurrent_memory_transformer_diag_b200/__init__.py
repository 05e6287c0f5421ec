"""B200-native (sm_100a) Diagonal Batching forward of a layer-recurrent
associative memory transformer (ARMT).

The compute lives in ``libarmt.so`` (C ABI: ``include/armt.h``); this package
holds its ctypes binding (``armt``), the in-tree build (``build``) and the
seeded synthetic inputs (``inputs``).
"""
from .armt import Armt, ArmtError, grouped_gemm, lib, memory_write, memory_write_static  # noqa: F401
from .inputs import CONFIGS, ArmtConfig, make_embeddings, make_weights  # noqa: F401
