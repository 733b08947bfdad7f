"""CPU oracle for SharQ's online sparse-dense activation decomposition.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, obviously correct
numpy restatement of what the GPU path computes.  Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it.  The product path (the CUDA library and its
Python binding) never imports it and shares no code with it.

Source of the method: "SharQ: Bridging Activation Sparsity and FP4 Quantization
for LLM Inference" (arXiv 2606.26587), as described on the xllm-io paper review
(sections 3.1-3.6) and the kasblo.com explainer (sections on NVFP4, 4:8
in-pairs and the residual).  Every function cites the passage it follows.

Parity status per function (details in each docstring):
  formats.e2m1_*     pinned: exhaustive table + ml_dtypes cross-check
  formats.e4m3_*     pinned: exhaustive table + torch/ml_dtypes cross-check
  formats.bf16_round pinned: torch bf16 cast cross-check
  sharq.rmsnorm      pinned: closed form + torch rms_norm cross-check
  sharq.pts_scale    pinned: closed form
  sharq.pair_mask    pinned: brute force over all score 4-tuples
  sharq.nvfp4_quant  pinned: round-trip closed forms, error bound
  sharq.prep         pinned: residual identity, worked example, bound
  sharq.pack_weight  pinned: duplication and round-trip bound
  sharq.linear       pinned: pure-python loop on tiny shapes, error bound
"""
