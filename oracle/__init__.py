"""CPU oracle for the BigBird ITC block-sparse attention forward pass.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call, link or
execute anything in this package: only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference leg of ``bench.py`` use it. The oracle shares
no code with the CUDA path (``block_sparse_long_attention_b200``); it does not
import that package and that package does not import this one.

Page abbreviations used in the citations of this package:

* [TFG-BigBird] -- the article "models 仓库中的 BigBird：线性复杂度稀疏注意力与长序列
  训练的完整实践" (TensorFlow Model Garden ``official/projects/bigbird``).
* [HF-Pegasus] -- the article "BigBirdPegasus 长序列条件生成模型详解从稀疏注意力原理到
  Transformers 实战" (Hugging Face ``modeling_bigbird_pegasus.py``).
"""

from .bigbird_oracle import (  # noqa: F401
    BIAS_MASKED,
    attention,
    attention_backward,
    attention_lse,
    attention_probs,
    attention_probs_rows,
    attention_rows,
    backward_flops,
    block_mask,
    brute_force_rows,
    check_shape,
    is_fallback,
    keys_per_row,
    mask_prep,
    pattern_table,
    rand_attn_generate,
    rand_attn_validate,
    sparse_flops,
    splitmix64_mix,
    splitmix64_output,
)
