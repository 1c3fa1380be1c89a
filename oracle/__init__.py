"""Float64 CPU oracle for one Psi-Spec decode step (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The CUDA library and its Python binding
never import it, and it imports nothing from them.
"""

from .uno_oracle import (  # noqa: F401
    PHILOX_WORD_ACCEPT,
    PHILOX_WORD_DRAFT,
    PHILOX_WORD_SAMPLE,
    bf16_bits_to_f64,
    draft_uniforms,
    dualpath_linear,
    philox4x32_10,
    round_to_bf16,
    sample_drafts,
    sample_drafts_u,
    softmax_rows,
    uniforms_for_block,
    merge_row_stats,
    row_stat_partials,
    verify_block,
    verify_block_head,
    verify_block_u,
    word_to_uniform,
)
from .tree_sampler import (  # noqa: F401,E402
    tree_build,
    tree_candidates,
    tree_draft,
    tree_max_nodes,
    tree_topk,
    tree_uniforms,
    tree_verify,
    tree_verify_u,
)
