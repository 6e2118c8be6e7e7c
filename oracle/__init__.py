"""Plain fp64 CPU oracle for the FVAttn routing front end and block-sparse attention.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it. It shares no code with the
CUDA library (``block_sparse_attention_video_b200``) and imports nothing from it.

Sources (page title, section):
  [FVAttn] "FVAttn: Adaptive Sparse Attention with Runtime Load Balancing for
           Video Generation" (Liu et al.), read through its Chinese translation,
           its English summary and its abstract page.
  [GSRS]   "Sparse Attention for Video Generation Acceleration via Growing
           Sparsity and Reduced Search".
  [LVSA]   "LVSA: Training-Free Sparse Attention for Long Video Diffusion".
"""

from .fvattn_oracle import (  # noqa: F401
    num_blocks,
    tile_order,
    permute,
    inverse_permute,
    block_mean_pool,
    block_scores,
    topp_topk_select,
    route,
    selection_mask,
    head_work,
    masked_attention,
    masked_attention_rows,
    dense_attention,
)
from .gsrs_oracle import (  # noqa: F401
    block_lse_rows,
    row_lse,
    block_importance_row,
    block_importance,
    attention_recall,
)
from .lvsa_oracle import (  # noqa: F401
    global_frames,
    attended_frames,
    frame_mask,
    lvsa_block_mask,
)
from .lowprec_oracle import (  # noqa: F401
    e4m3_encode,
    e4m3_decode,
    quantize_v,
    dequantize_v,
    masked_attention_qv,
    masked_softmax_weights,
)
from .hilbert_oracle import (  # noqa: F401
    hilbert_index,
    hilbert_order,
)
from .mask_parity import (  # noqa: F401
    BORDER_REL,
    BORDER_CUM,
    compare_masks,
    borderline_ceiling,
)
