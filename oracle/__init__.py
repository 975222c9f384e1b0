"""CPU oracle for MHA2MLA conversion and latent-cache decode — TEST INFRASTRUCTURE ONLY.

Plain float64 numpy (LAPACK SVD, BLAS matmul as library steps), written from the
method's definitions and sharing no code with the CUDA path.  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
it; the product library never calls it and has no CPU fallback.

Every function cites the passage it follows.  Page short names:
  NOTES  = "MHA2MLA: Towards Economical Inference by Enabling DeepSeek's Multi-Head
           Latent Attention in Any Transformer-based LLMs" (paper notes, ACL 2025);
           sections 方法详解/整体框架 (overall framework), 关键设计 (key designs:
           contribution-aware partial-RoPE removal; joint SVD low-rank approximation
           (SVDjoint); compatibility with KV-cache quantization), 实验关键数据 (tables).
  ABSTRACT = arXiv record "Towards Economical Inference: Enabling DeepSeek's Multi-Head
           Latent Attention in Any Transformer-based LLMs", abstract.
  SUMMARY = "What is MHA2MLA" product page, §Technical principles.
  README = GitHub README "MHA2MLA", §Fine-Tuning (strategy tables), §LongBench
           Evaluation (quantized cache).

Pinning status (see tests/test_oracle_pins.py):
  pair_scores, select_pairs, split_dims, svd_joint, krope_weights, rotate, append,
  decode_unabsorbed, decode_absorbed, mha_textbook_* — pinned by closed forms,
  brute force, invariants and hand-derived fixtures.
  quant_int4_g32 / dequant_int4_g32 — the scheme itself is a reading (the pages
  name 4-bit quantization of the latent but not its encoding); the oracle's
  implementation of that reading is pinned by its error bound, exact round trips and
  hand-derived codes.
  cache_bytes_per_token — pinned by the pages' printed reduction figures under a
  stated reading of the unstated configuration.
  fixed_pairs — the pages name the high / low / uniform / full strategies without
  formulas; the reading is pinned by its frequency meaning (rope_theta ordering),
  hand-written sets and the full-RoPE case, which reduces to textbook RoPE MHA.
  quant_int2_g32 / dequant_int2_g32 / pack_int2 — the Notes name 2-bit quantisation of
  the latent without an encoding; the reading (the int4 scheme at 2 bits) is pinned by
  its error bound, the group maximum landing on +-1, exact round trips, hand-derived codes
  and a hand-derived byte.
  residual_window — the README gives only the residual length (128) of the quantised
  cache; the reading (the most recent tokens read unquantised) is pinned by its special
  cases (no window: the int4 values; a window over the whole sequence: the plain values),
  by a brute-force ring-with-position-tags model for in-order appends, and by the decodes
  it reduces to.
"""

from .mha2mla import *  # noqa: F401,F403
