"""Float64 CPU oracle for the MoBA causal prefill forward, its decode step, the min/max gate
variant and the backward pass.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this package: only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code, table or constant with the CUDA path under
``block_sparse_long_meanpool_b200/``.

Every function follows the plain definition of the method as stated on the
page "《MoBA: Mixture of Block Attention for Long-Context LLMs》深度解读报告"
(the zako-mio knowledge-base analysis of the MoBA paper), sections 2.1-2.3 and
3.2 (2.5 for the backward's treatment of the parameter-free gate; 1.3, 5.1 and 6.3 for the
min/max variant, whose formula is Quest's), and on the course page "Paper: MoBA (Moonshot)"
(module F26).  Where those pages are silent the reading taken is stated in the docstring.

Parity pins: every function here is pinned by a ``-m "not gpu"`` test in
``tests/test_oracle_pins.py`` against something other than itself (a library
routine it reduces to, torch autograd, finite differences, brute force, closed forms,
the pages' printed sparsity figures).  No function is "parity unpinned".
"""

from .moba_ref import (  # noqa: F401
    block_table,
    block_means,
    block_minmax,
    minmax_scores_row,
    gate_scores_row,
    select_blocks,
    select_blocks_rows,
    attend_rows,
    attention_masked_dense,
    moba_forward,
    moba_backward,
    moba_decode,
    attended_keys,
)
