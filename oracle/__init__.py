"""CPU oracle for the contextual-token-sparsity hot path (test infrastructure).

This package is the correctness reference for the CUDA library and nothing
else: only the tests, the package smoke check and the benchmark's CPU-baseline
leg may import it. It shares no code with the CUDA path (no kernels, headers,
helpers or tables), computes in float64 from the same bf16 bytes, and follows
the definitions of

* "Jenga: Enhancing LLM Long-Context Fine-tuning with Contextual Token
  Sparsity" (aipaper.cc summary of the USENIX ATC'25 paper), §4.2.1 Eq. 1,
  Eq. 2, Fig. 6 and the layer-specific-threshold paragraph; §4.2.2 Eq. 3;
  §4.2.3 "Permutation-free Token Movement" (selective load, in-place addition)
  and "Segment-based Peak Cutting";
* "LeMo" (pith.science reading of arXiv 2501.09767), "What carries the
  argument".

Every function states the passage it follows and, where the pages are silent,
the reading taken.  See ``oracle.lemo_oracle`` for the functions.
"""

from .lemo_oracle import (  # noqa: F401
    bf16_bits_to_f64,
    f64_to_bf16_bits,
    block_max_row,
    score_blocks,
    column_scores,
    threshold_for_keep_ratio,
    keep_mask,
    compact,
    gather_pad,
    scatter_residual,
    block_representatives,
    predictor_embeddings,
    predict_scores,
    recall,
    recompute_input,
    mlp_token_scores,
    mlp_block_scores,
    lm_head_loss,
    lm_head_loss_f64,
    lm_head_rows,
    attention_kept,
    attention_residual_exact,
    attention_kept_rows,
)
