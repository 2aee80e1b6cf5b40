"""CPU oracle for layer-streamed LoRA training over a frozen NF4 base.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library under
``layer_streamed_qlora_b200/`` and its Python binding) imports, links or calls
this package; only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code, table or helper with the CUDA path; the one shared module is
``soup_synth`` (seeded random inputs, none of the method's arithmetic).

What it computes, and where that is defined
-------------------------------------------
Layer streaming and checkpoint recompute are exact reorderings of ordinary
LoRA training (the Soup pages, "how layer streaming works": each decoder layer
is read once in the forward pass and once more for the recompute, because the
gradient to the layer below needs dL/dx = W^T dL/dy with W frozen).  So the
oracle is the plain, unstreamed, unrecomputed definition, differentiated by
hand with the chain rule written out per operation (no autograd):

* ``oracle.nf4``   - NF4 block quantisation and dequantisation (QLoRA's
  NormalFloat-4 data type; 64-element blocks, fp32 absmax, 2 codes per byte).
* ``oracle.lora``  - a LoRA linear layer y = W x + (alpha/r) B A x and its
  backward pass with W frozen.
* ``oracle.layer`` - one Llama-style decoder layer (RMSNorm, RoPE, causal GQA
  attention, SwiGLU) with LoRA on all seven projections, forward and backward.
* ``oracle.head``  - token embedding, final norm, lm_head, next-token
  cross-entropy, sequence log-probabilities and the DPO loss.
* ``oracle.model`` - the whole stack for one SFT or DPO step.

Floating point is fp64 throughout, except where the method itself fixes a
precision: NF4 quantisation and dequantisation are defined in fp32 with a final
round-to-nearest-even to bf16, and every operand the GPU receives (activations,
LoRA factors, dequantised weights) is a bf16 value, which the oracle takes as
the exact fp64 number it represents.

Parity pins: every function here is checked by ``tests/test_oracle_*.py``
against closed forms, invariants, special cases, finite differences and brute
force; none of those checks re-types the function it checks.
"""
