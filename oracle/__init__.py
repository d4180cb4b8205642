"""CPU oracle for the token-sparse layer path -- TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously-correct numpy (float64) restatement of what the path
computes, written from the Jenga paper ("Jenga: Enhancing LLM Long-Context
Fine-tuning with Contextual Token Sparsity", ATC'25) as described on two pages:
the papercache.org deep notes ("Jenga notes") and the aipaper.cc summary ("Jenga
summary").  Every function cites the section / equation it follows.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (``token_sparse_long_b200``)
never imports it and shares no code with it: no kernels, headers, helpers, tables
or constant generators.  The two sides meet only in the seeded input generators
of ``synth`` (which hold none of the method's arithmetic).

Modules
-------
bf16       round-to-nearest-even float64 -> bf16 (storage rounding at stated points)
scores     block informativeness (softmax column mass; Eq. 2 block-max form)
select     threshold selection / top-k / compaction to ascending block indices
movement   permutation-free gather and in-place scatter-add
lm_loss    causal-LM cross-entropy over the vocabulary and its hidden-state gradient
mlp_blocks MLP-block elimination criterion (|SiLU(gate) * up| mass per block) and index composition
layer      retained-token Llama decoder layer forward and backward (+ segmented)
predictor  block-score predictor MLP (mean pool -> Linear -> GELU -> Linear)
rank       rank agreement statistics (Spearman, Kendall tau-b, top-k recall)

Parity status: every function is pinned by ``tests/test_oracle_*.py`` except the
accuracy claims of the paper (PPL, predictor recall on real data), which need
trained weights and datasets and are "parity unpinned".
"""
