"""CPU oracle for block-sparse video attention (TEST INFRASTRUCTURE ONLY).

Plain, slow, fp64 numpy restatements of what the hot path computes, written
from the pages' descriptions of the methods:

* LiteAttention write-up (arXiv 2511.11062), sections 3, 5 and 6 (skip rule,
  persistent skip mask carried across denoising steps);
* VMoBA write-up (arXiv 2506.23858), the "threshold dynamic selection" and
  "global block selection" paragraphs (mean-pooled block scores, cumulative
  threshold selection);
* "MIT实验室推出Radial Attention" (arXiv 2506.19852), the exponential
  spatio-temporal decay and static-mask paragraphs;
* "浙江大学突破视频AI瓶颈:金字塔方法提升视频AI效率10倍" (PSA, arXiv
  2512.04025), the pyramid KV, multi-level mask and distribution-consistent
  attention paragraphs;
* PAROAttention write-up (pattern-aware reordering) and VMoBA's recurrent
  1D / 2D / 3D partitions: token permutations of the grid, ``oracle/permute.py``;
* the backward pass (gradients through the masked attention, needed by the
  Radial Attention write-up's LoRA length extension) is the derivative of
  the forward definition, stated in ``oracle/backward.py``.

The pages give prose only; the concrete rules (tau-mass selection, radial
window S / 2^floor(log2 dt), skip test with epsilon in natural-log logits,
ln(pool count) bias) are the plainest readings stated in each function.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  It shares
no code with the CUDA library and never imports it.
"""
from .attention import masked_attention, dense_attention, block_mask_to_token_mask
from .masks import block_means, block_scores, tau_mask, level_map, radial_mask, global_mask
from .pyramid import pyramid_pool, pyramid_attention
from .lite import lite_step, lite_chain, visit_order, skip_flags
from .backward import masked_attention_bwd, masked_attention_bwd_rows
from .permute import permutation, permute_tokens

__all__ = [
    "masked_attention", "dense_attention", "block_mask_to_token_mask",
    "block_means", "block_scores", "tau_mask", "level_map", "radial_mask", "global_mask",
    "pyramid_pool", "pyramid_attention", "lite_step", "lite_chain", "visit_order", "skip_flags",
    "masked_attention_bwd", "masked_attention_bwd_rows", "permutation", "permute_tokens",
]
