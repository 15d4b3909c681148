"""B200-native MoBA (Mixture of Block Attention): the causal prefill forward and its backward
pass, the decode step with the mean or the min/max block gate.

The compute path is the C-ABI library ``libmoba.so`` (CUDA for sm_100a, headers in
``include/moba.h``); ``moba`` is its thin ctypes binding and ``workloads`` makes seeded
synthetic inputs.  Build the library with ``python -m block_sparse_long_meanpool_b200.build``.
"""

from .moba import (  # noqa: F401
    MobaError,
    attn_bwd,
    attn_fwd,
    decode_fwd,
    decode_minmax_fwd,
    gate_topk,
    load_library,
    make_params,
    meanpool,
    minmaxpool,
    num_blocks,
    workspace_size,
)
